// pair_kernel.cuh -- the reused denoising step, and the plan's residual pass,
// run over PAIRS of adjacent query groups that share one list of gathered keys.
//
// Groups 2p and 2p+1 of a head are neighbours in the grouping order (cctest.ai,
// "MC-Sparse Narrows the Dense-Sparse Attention Gap in Diffusion Transformers",
// "Hardware-aware query organization": similar queries are organised into
// tile-aligned groups), so they keep mostly the same KV tokens (about 80 % of
// the k kept keys on the DiT-shaped layers this library is measured on).  The
// step is bound by gathering index-listed K/V rows (cnshai.top post, "What
// Trips People Up": irregular gathers are what tile-aligned grouping pays for),
// so a pair is served from ONE list: the union of the two groups' kept keys,
// ordered [keys only group 2p keeps | keys both keep | keys only 2p+1 keeps].
// Group 2p's keys are then the union positions [0, k) and group 2p+1's the
// positions [u - k, u) (u = union size): each group attends to a contiguous
// range of the gathered tiles, masked only on the tiles at its range's ends,
// and the keys both keep are gathered once for both.  The result per group is
// exactly its own sparse attention (attention over a set of keys does not
// depend on their order); only fp32 summation order differs from the
// one-group kernel in attn_kernel.cuh.
//
//  kModeStep      O_i = softmax over the group's kept keys of (scale Q_i.K_j)
//                 applied to V, plus the cached residual R_i; bf16 out
//                 (aiqbench.com abstract: groups, KV indices and residuals
//                 "reused across subsequent denoising steps").
//  kModePlanResid R_i = O_dense_i - O_sparse_i with O_dense from the plan's
//                 statistics pass ("residuals between dense and sparse
//                 attention outputs").
//
// CTA (persistent, one per SM) = items (head, pair), head-major; per item the
// union's key tiles of 64:
//   warps 0-3  softmax group A: query rows of group 2p       (S_A0, S_A1, O_A)
//   warps 4-7  softmax group B: query rows of group 2p+1     (S_B0, S_B1, O_B)
//              thread t owns query row t % 128 (TMEM lane); rows past the
//              group's size are padding (computed on a valid row, never written)
//   warp  8    TMEM allocation and the single UMMA-issuing thread
//   warps 9-12 K-ring TMA tile::gather4 producers
//   warps 13-15 V-ring producers, which also gather each item's two Q tiles
// The softmax warpgroups take more registers than the rest (setmaxnreg).
// TMEM: per group two S buffers of 64 columns and O (D columns): 4 x 64 + 2 D
// <= 512 columns.  Key tiles of 64 (not 128) are what let each group keep a
// double-buffered S next to its O: Q.K^T of a group's tile j+2 is issued
// right after its P.V(j), so its softmax finds the next S ready and runs
// back to back.  P (bf16 hi and lo parts, two P.V MMAs, ~2^-17 relative
// error) is written over its own S buffer: hi pairs in columns [0, 32), lo
// pairs in [32, 64).  The tensor pipe interleaves the groups per tile:
//   P.V_A(j), Q.K^T_A(j+2), P.V_B(j), Q.K^T_B(j+2), ...
// "S full", "P ready" and "P.V done" barriers alternate by the parity of the
// group's own tile count, so each has at most one phase outstanding (P of
// tile i+2 needs S of i+2, whose Q.K^T is issued after P.V(i), which needs P
// of tile i).  A softmax warp waits for the previous P.V only when a row's
// max moved by more than 2^32 (the lazy rescale of O) and in the epilogue.
// Every wait is bounded; out-of-range indices are never gathered.
#pragma once

#include "attn_kernel.cuh"

namespace mcs {

template <int D>
struct PairCfg {
  static constexpr int BM = 128, BN = 64;       // query rows per group block, keys per tile
  static constexpr int NK = D == 64 ? 10 : 5;   // K ring depth (tiles)
  static constexpr int NV = D == 64 ? 10 : 5;   // V ring depth
  static constexpr int Q_BYTES = BM * D * 2;    // one query block
  static constexpr int KV_BYTES = BN * D * 2;   // one key tile
  static constexpr int OFF_Q = 0;               // Q_A, then Q_B
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NV * KV_BYTES;
  // per block q full/empty, k/v full/empty, per group s_full[2], p[2], pv[2], drain
  static constexpr int N_BAR = 4 + 2 * NK + 2 * NV + 12 + 1;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BAR;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;   // + slack to align the base to 1 KB
  static constexpr int MMA_WARP = 8, KW = 4, VW = 3;
  static constexpr int THREADS = (9 + KW + VW) * 32;   // 512
  // registers per thread after the split: 256 softmax threads x 160 +
  // 256 other threads x 96 = 65536, the launch's 512 x 128
  static constexpr int REG_SOFTMAX = 160, REG_OTHER = 96;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0;            // S of group X, buffer b: X * 128 + b * 64
  static constexpr uint32_t COL_O_A = 256, COL_O_B = 256 + D;
  static constexpr float kRaise = 32.f;   // lazy rescale bound, as in attn_kernel.cuh
};
static_assert(PairCfg<128>::SMEM <= 232448 && PairCfg<64>::SMEM <= 232448, "shared memory budget");
static_assert(PairCfg<128>::REG_SOFTMAX * 256 + PairCfg<128>::REG_OTHER * 256 <= 65536, "register split");

// BLOCK = 0: the union lists hold individual keys, gathered row by row.
// BLOCK = 64 or 128: they hold indices of aligned blocks of BLOCK keys (a
// block-sparse selection, the comparison point of block-granular methods);
// each 64-key tile is then one contiguous TMA tile load per column block, by
// one lane, and no tile is partial.  Everything past the producers works in
// key positions, so the rest of the kernel is the same.
template <int D, int MODE, int BLOCK = 0>
__global__ void __launch_bounds__(PairCfg<D>::THREADS, 1) pair_kernel(const __grid_constant__ AttnArgs a) {
  static_assert(MODE == kModeStep || MODE == kModePlanResid, "sparse modes only");
  static_assert(BLOCK == 0 || BLOCK == 64 || BLOCK == 128, "blocks of 64 or 128 keys");
  using C = PairCfg<D>;
  constexpr int BM = C::BM, BN = C::BN, NK = C::NK, NV = C::NV;
  constexpr int NDB = D / 64;                       // 64-column (128-byte) blocks per row
  constexpr uint32_t Q_TX = BM * D * 2u;            // bytes of one query block
  constexpr uint32_t TILE_TX = BN * D * 2u;         // bytes of one key tile

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ0 = sbase + C::OFF_Q;
  const uint32_t sK0 = sbase + C::OFF_K;
  const uint32_t sV0 = sbase + C::OFF_V;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  // the query block of group X: loaded (q full), read by its item's last Q.K^T (q empty)
  auto b_q = [&](int X) { return bar0 + 8 * X; };
  auto b_qempty = [&](int X) { return bar0 + 16 + 8 * X; };
  auto b_kfull = [&](int s) { return bar0 + 8 * (4 + s); };
  auto b_kempty = [&](int s) { return bar0 + 8 * (4 + NK + s); };
  auto b_vfull = [&](int s) { return bar0 + 8 * (4 + 2 * NK + s); };
  auto b_vempty = [&](int s) { return bar0 + 8 * (4 + 2 * NK + NV + s); };
  const uint32_t bx = bar0 + 8 * (4 + 2 * NK + 2 * NV);
  // per group X and tile-count parity b
  auto b_sfull = [&](int X, int i) { return bx + 8 * (X * 6 + (i & 1)); };
  auto b_p = [&](int X, int i) { return bx + 8 * (X * 6 + 2 + (i & 1)); };
  auto b_pv = [&](int X, int i) { return bx + 8 * (X * 6 + 4 + (i & 1)); };
  const uint32_t b_drain = bx + 8 * 12;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int N = a.N;
  const int k_units = a.k;            // list entries per group: keys, or blocks
  const int kk = BLOCK ? k_units * BLOCK : k_units;   // keys per group, <= N
  const int n_pairs = a.n_pairs;
  const int n_items = a.BH * n_pairs;
  const int a_tiles = (kk + BN - 1) / BN;   // group A's tiles: [0, a_tiles)

  // One item: (head, pair).  Union list of u keys; group A = 2p keeps union
  // positions [0, k), group B = 2p+1 (absent past the head's last group)
  // keeps [u - k, u).  Tiles of the union: T; B's tiles [b0, T).
  struct Item {
    int bh, p, u, T, b0;
    bool hasB;
    size_t head;
    const int32_t *list;
  };
  auto item_at = [&](int item) -> Item {
    Item w;
    w.p = item % n_pairs;
    w.bh = item / n_pairs;
    w.head = static_cast<size_t>(w.bh) * N;
    w.list = a.pair_idx + (static_cast<size_t>(w.bh) * n_pairs + w.p) * (2 * static_cast<size_t>(k_units));
    w.hasB = 2 * w.p + 1 < a.n_groups;
    int u = a.pair_len[static_cast<size_t>(w.bh) * n_pairs + w.p];   // list entries
    const int umax = w.hasB ? 2 * k_units : k_units;
    if (u < k_units || u > umax) {   // corrupt metadata: never read past the list
      record_status(a.status, kStatusBadMeta);
      u = u < k_units ? k_units : umax;
    }
    w.u = BLOCK ? u * BLOCK : u;     // union positions, in keys
    w.T = (w.u + BN - 1) / BN;
    w.b0 = w.hasB ? (w.u - kk) / BN : w.T;
    return w;
  };
  // query row r of block X (0: group 2p, 1: group 2p+1) -> token, or -1 for padding
  auto q_raw = [&](const Item &w, int X, int r) -> int {
    const int gr = (2 * w.p + X) * a.G + r;
    return (r >= a.G || gr >= N || (X == 1 && !w.hasB)) ? -1 : a.perm[w.head + gr];
  };
  auto q_check = [&](int q) -> int {
    if (q != -1 && static_cast<unsigned>(q) >= static_cast<unsigned>(N)) {
      record_status(a.status, kStatusBadMeta);
      return -1;
    }
    return q;
  };

  if (tid == 0) {
    for (int X = 0; X < 2; ++X) {
      mbar_init(b_q(X), 1);
      mbar_init(b_qempty(X), 1);
    }
    for (int s = 0; s < NK; ++s) {
      mbar_init(b_kfull(s), 1);
      mbar_init(b_kempty(s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(b_vfull(s), 1);
      mbar_init(b_vempty(s), 1);
    }
    for (int X = 0; X < 2; ++X)
      for (int i = 0; i < 2; ++i) {
        mbar_init(b_sfull(X, i), 1);
        mbar_init(b_p(X, i), 128);
        mbar_init(b_pv(X, i), 1);
      }
    mbar_init(b_drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::MMA_WARP + 1 && lane == 0) {
    tma_prefetch_desc(&a.tmQ);
    tma_prefetch_desc(&a.tmK);
    tma_prefetch_desc(&a.tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp > C::MMA_WARP) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REG_OTHER));
    // ------------------------------------------------------------------ TMA producers
    const int pw = warp - C::MMA_WARP - 1;    // 0..KW-1: K ring, KW..KW+VW-1: V ring (+ Q)
    const bool is_k = pw < C::KW;
    const int NW = is_k ? C::KW : C::VW;
    const int h = is_k ? pw : pw - C::KW;
    const void *tm = is_k ? static_cast<const void *>(&a.tmK) : static_cast<const void *>(&a.tmV);
    const int NS = is_k ? NK : NV;
    const uint32_t ring = is_k ? sK0 : sV0;
    // gather4 operation o (4 rows x 128 bytes) of a key tile belongs to warp
    // o % NW, lane o / NW; a tile has BN / 4 row quads x NDB column blocks
    constexpr int OPS = (BN / 4) * NDB;
    const int op_raw = h + NW * lane;
    const bool active = op_raw < OPS;
    const int op = active ? op_raw : h;
    const int quad = op % (BN / 4), dbk = op / (BN / 4);
    bool ok = true;
    int issued = 0;                           // fills of this ring by this CTA
    int nqX[2] = {0, 0};                      // Q loads per block (V-ring warps)
    // The row indices of a tile come from the union list in global memory;
    // the list loads of the next R tiles are kept in flight (one register set
    // per tile, the loop unrolled by R so each set stays in registers), so a
    // tile's gathers never wait a memory round trip for their indices.
    constexpr int R = 4;
    Item w;
    if (static_cast<int>(blockIdx.x) < n_items) w = item_at(blockIdx.x);
    for (int item = blockIdx.x, it = 0; item < n_items && ok; item += gridDim.x, ++it) {
      const int nitem = item + static_cast<int>(gridDim.x);
      Item wn = w;
      if (nitem < n_items) wn = item_at(nitem);      // its list length is loaded during this item
      const int first = w.list[0];
      auto tile_rows = [&](int t, int (&rows)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int pos = t * BN + 4 * quad + i;
          rows[i] = pos < w.u ? w.list[pos] : first;   // past the union: re-read a kept key (masked)
        }
      };
      auto checked = [&](int key) -> int {
        if (static_cast<unsigned>(key) >= static_cast<unsigned>(N)) {
          record_status(a.status, kStatusBadMeta);
          key = 0;
        }
        return static_cast<int>(w.head) + key;
      };
      int pre[R][4];
#pragma unroll
      for (int s = 0; s < R; ++s)
        if (BLOCK == 0 && active && s < w.T) tile_rows(s, pre[s]);
      if (!is_k) {
        // each group's query block, once that group's last Q.K^T of its
        // previous item has read the buffer; the rows are looked up first
        constexpr int QOPS = (BM / 4) * NDB;
#pragma unroll
        for (int X = 0; X < 2; ++X) {
          if (!ok) break;
          if (X == 1 && !w.hasB) continue;
          int qr[2][4];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int o = h + NW * lane + u * NW * 32;
            const int qd = o % (BM / 4);
            if (o < QOPS) {
              const int q0 = q_check(q_raw(w, X, 0));
              const int fb = q0 >= 0 ? q0 : 0;          // padding rows re-read a valid row
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int q = q_check(q_raw(w, X, 4 * qd + i));
                qr[u][i] = static_cast<int>(w.head) + (q >= 0 ? q : fb);
              }
            }
          }
          if (nqX[X] > 0) {
            int got = 1;
            if (lane == 0) got = mbar_wait(b_qempty(X), (nqX[X] - 1) & 1, a.wait_ns, abort_flag);
            got = __shfl_sync(0xffffffffu, got, 0);
            if (!got) { ok = false; break; }
          }
          if (h == 0 && lane == 0) mbar_arrive_expect_tx(b_q(X), Q_TX);
          __syncwarp();
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int o = h + NW * lane + u * NW * 32;
            if (o < QOPS) {
              const int qd = o % (BM / 4), db = o / (BM / 4);
              tma_gather4(sQ0 + X * C::Q_BYTES + db * (BM * 128) + qd * 512, &a.tmQ, db * 64, qr[u][0], qr[u][1],
                          qr[u][2], qr[u][3], b_q(X));
            }
          }
          ++nqX[X];
        }
        if (!ok) break;
      }
      if constexpr (BLOCK != 0) {
        // contiguous blocks: one lane of the ring's first warp loads each
        // 64-key tile as NDB tile boxes of 64 rows
        for (int j = 0; j < w.T && ok && h == 0; ++j) {
          const int slot = issued % NS;
          int got = 1;
          if (lane == 0)
            got = mbar_wait(is_k ? b_kempty(slot) : b_vempty(slot), ((issued / NS) & 1) ^ 1, a.wait_ns,
                            abort_flag);
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) { ok = false; break; }
          if (lane == 0) {
            const uint32_t full = is_k ? b_kfull(slot) : b_vfull(slot);
            const uint32_t dst = ring + slot * C::KV_BYTES;
            int blk = w.list[(j * BN) / BLOCK];
            if (static_cast<unsigned>(blk) >= static_cast<unsigned>(N / BLOCK)) {   // corrupt metadata
              record_status(a.status, kStatusBadMeta);
              blk = 0;
            }
            const int row = static_cast<int>(w.head) + blk * BLOCK + (j * BN) % BLOCK;
            mbar_arrive_expect_tx(full, TILE_TX);
#pragma unroll
            for (int db = 0; db < NDB; ++db) tma_load_2d(dst + db * (BN * 128), tm, db * 64, row, full);
          }
          __syncwarp();
          ++issued;
        }
      } else {
      for (int jb = 0; jb < w.T && ok; jb += R) {
#pragma unroll
        for (int s = 0; s < R; ++s) {
          const int j = jb + s;
          if (j >= w.T || !ok) break;
          const int slot = issued % NS;
          int got = 1;
          if (lane == 0)
            got = mbar_wait(is_k ? b_kempty(slot) : b_vempty(slot), ((issued / NS) & 1) ^ 1, a.wait_ns,
                            abort_flag);
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) { ok = false; break; }
          const uint32_t full = is_k ? b_kfull(slot) : b_vfull(slot);
          const uint32_t dst = ring + slot * C::KV_BYTES;
          // one expect-tx arrival per phase; the other warps' bytes may land first
          if (h == 0 && lane == 0) mbar_arrive_expect_tx(full, TILE_TX);
          __syncwarp();
          if (active) {
            tma_gather4(dst + dbk * (BN * 128) + quad * 512, tm, dbk * 64, checked(pre[s][0]), checked(pre[s][1]),
                        checked(pre[s][2]), checked(pre[s][3]), full);
            if (j + R < w.T) tile_rows(j + R, pre[s]);   // R tiles ahead, into the set just used
          }
          ++issued;
        }
      }
      }
      w = wn;
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
      for (int X = 0; X < 2 && !is_k; ++X)
        if (nqX[X] > 0) mbar_wait(b_q(X), (nqX[X] - 1) & 1, 2000000000ull, &never);
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REG_OTHER));
    // ------------------------------------------------------------------ UMMA issue
    {   // the whole warp runs the loop; one elected lane issues each tcgen05 instruction
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, 1);
      bool ok = true;
      int gt = 0;                 // key tiles of earlier items (ring slots and phases)
      int cnt[2] = {0, 0};        // each group's tiles before this item (S buffers, phases)
      int nqm[2] = {0, 0};        // query blocks consumed per group
      for (int item = blockIdx.x, it = 0; item < n_items && ok; item += gridDim.x, ++it) {
        const Item w = item_at(item);
        const int T = w.T;
        const int j0B = w.b0;
        auto act = [&](int X, int j) -> bool { return X == 0 ? j < a_tiles : (j >= j0B && j < T); };
        // the group's own tile count at tile j of this item
        auto idx = [&](int X, int j) -> int { return X == 0 ? cnt[0] + j : cnt[1] + (j - j0B); };
        // Q.K^T of tile j for group X; K slot released after the tile's last one
        auto issue_qk = [&](int j, int X) -> bool {
          const int gj = gt + j;
          const int s = gj % NK;
          const bool first = X == 0 || !act(0, j);
          const bool last = X == 1 || !act(1, j);
          if (j == (X == 0 ? 0 : j0B)) {   // the group's first tile: its query block
            if (!mbar_wait_warp(b_q(X), nqm[X] & 1, a.wait_ns, abort_flag)) return false;
            ++nqm[X];
          }
          if (first) {
            if (!mbar_wait_warp(b_kfull(s), (gj / NK) & 1, a.wait_ns, abort_flag)) return false;
          }
          tc_fence_after();
          const int i = idx(X, j);
          const uint32_t tS = tbase + C::COL_S + X * 128 + (i & 1) * BN;
          // descriptors advance by (byte offset >> 4) in their address field
          const uint64_t dq = sdesc_sw128(sQ0 + X * C::Q_BYTES, 16, 1024);
          const uint64_t dk = sdesc_sw128(sK0 + s * C::KV_BYTES, 16, 1024);
#pragma unroll
          for (int k16 = 0; k16 < D / 16; ++k16) {
            const uint32_t qoff = ((k16 >> 2) * (BM * 128) + (k16 & 3) * 32) >> 4;
            const uint32_t koff = ((k16 >> 2) * (BN * 128) + (k16 & 3) * 32) >> 4;
            umma_bf16_ss_elect(tS, dq + qoff, dk + koff, idesc_qk, k16 > 0 ? 1u : 0u);
          }
          umma_commit_elect(b_sfull(X, i));
          if (j == (X == 0 ? a_tiles : T) - 1) umma_commit_elect(b_qempty(X));   // the group's last read of Q
          if (last) umma_commit_elect(b_kempty(s));
          return true;
        };
        // P.V of tile j for group X; V slot released after the tile's last one
        auto issue_pv = [&](int j, int X) -> bool {
          const int gj = gt + j;
          const int s = gj % NV;
          const bool first = X == 0 || !act(0, j);
          const bool last = X == 1 || !act(1, j);
          const int i = idx(X, j);
          if (!mbar_wait_warp(b_p(X, i), (i >> 1) & 1, a.wait_ns, abort_flag)) return false;
          if (first && !mbar_wait_warp(b_vfull(s), (gj / NV) & 1, a.wait_ns, abort_flag)) return false;
          tc_fence_after();
          const uint32_t tP = tbase + C::COL_S + X * 128 + (i & 1) * BN;
          const uint32_t tO = tbase + (X ? C::COL_O_B : C::COL_O_A);
          const uint64_t dv = sdesc_sw128(sV0 + s * C::KV_BYTES, BN * 128, 1024);
          const bool first_of_item = j == (X == 0 ? 0 : j0B);
#pragma unroll
          for (int k16 = 0; k16 < BN / 16; ++k16)   // hi parts
            umma_bf16_ts_elect(tO, tP + 8 * k16, dv + ((k16 * 16 * 128) >> 4), idesc_pv,
                         (!first_of_item || k16 > 0) ? 1u : 0u);
#pragma unroll
          for (int k16 = 0; k16 < BN / 16; ++k16)   // lo parts
            umma_bf16_ts_elect(tO, tP + 32 + 8 * k16, dv + ((k16 * 16 * 128) >> 4), idesc_pv, 1u);
          umma_commit_elect(b_pv(X, i));
          if (last) umma_commit_elect(b_vempty(s));
          return true;
        };
        // the first two tiles' Q.K^T of each group, in tile order (the group
        // loops are unrolled so each group's counters stay in registers)
        ok = true;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int X = 0; X < 2; ++X)
            if (ok && act(X, j)) ok = issue_qk(j, X);
        for (int j = 0; j < T && ok; ++j) {
#pragma unroll
          for (int X = 0; X < 2; ++X) {
            if (ok && act(X, j)) ok = issue_pv(j, X);
            if (ok && j + 2 < T && act(X, j + 2)) ok = issue_qk(j + 2, X);
          }
        }
        cnt[0] += a_tiles;
        cnt[1] += T - j0B;
        gt += T;
      }
      if (!ok && lane == 0 && !*abort_flag) {
        *abort_flag = 1;
        record_status(a.status, kStatusTimeout);
      }
      // make sure nothing issued is still running before TMEM is released
      umma_commit_elect(b_drain);
      volatile int never = 0;
      mbar_wait_warp(b_drain, 0, 2000000000ull, &never);
      __syncwarp();
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REG_SOFTMAX));
    // ------------------------------------------------------------------ softmax groups (warps 0-7)
    const int X = warp >> 2;                          // 0: group 2p, 1: group 2p+1
    const int r = (warp & 3) * 32 + lane;             // query row == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS0 = tbase + lane_addr + C::COL_S + X * 128;
    const uint32_t tO = tbase + lane_addr + (X ? C::COL_O_B : C::COL_O_A);
    const float sl2 = a.scale_log2;
    // the epilogue's second input (residual, or the dense output), per row
    const float *ep_in = MODE == kModeStep ? a.residual : a.O32_in;
    // or a compact (bf16) residual; a reused step may add none (a block-sparse comparison)
    const bf16 *ep16 = MODE == kModeStep ? a.residual16 : nullptr;
    const bool has_res = ep_in != nullptr || ep16 != nullptr;
    constexpr int EC = 16;   // epilogue chunk (columns)
    // chunk cc of this row's epilogue input: 4 float4 of fp32, or (compact)
    // the 2 uint4 of its 16 bf16 values carried bit for bit in e[0], e[1]
    auto load_in = [&](size_t row, int cc, float4 (&e)[EC / 4]) {
      if (ep16 != nullptr) {
        const uint4 *src = reinterpret_cast<const uint4 *>(ep16 + row + cc * EC);
#pragma unroll
        for (int u = 0; u < EC / 8; ++u) {
          const uint4 t = __ldg(src + u);
          e[u] = make_float4(__uint_as_float(t.x), __uint_as_float(t.y), __uint_as_float(t.z), __uint_as_float(t.w));
        }
      } else {
        const float4 *src = reinterpret_cast<const float4 *>(ep_in + row + cc * EC);
#pragma unroll
        for (int u = 0; u < EC / 4; ++u) e[u] = __ldg(src + u);
      }
    };
    bool ok = true;
    int c = 0;       // this group's tiles so far (S buffer, barrier phases)
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const Item w = item_at(item);
      if (X == 1 && !w.hasB) continue;
      const int q = q_check(q_raw(w, X, r));
      const size_t row = (w.head + (q >= 0 ? q : 0)) * D;
      if (q >= 0 && has_res) {   // pull the epilogue row into L2 well before it is read
        if (ep16 != nullptr) {
#pragma unroll
          for (int cc = 0; cc < D / 64; ++cc) asm volatile("prefetch.global.L2 [%0];" ::"l"(ep16 + row + cc * 64));
        } else {
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) asm volatile("prefetch.global.L2 [%0];" ::"l"(ep_in + row + cc * 32));
        }
      }
      const int j0 = X == 0 ? 0 : w.b0;
      const int j1 = X == 0 ? a_tiles : w.T;
      // valid union positions of this group: [glo, ghi)
      const int glo = X == 0 ? 0 : w.u - kk;
      const int ghi = X == 0 ? kk : w.u;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = j0; j < j1; ++j, ++c) {
        if (!mbar_wait_warp(b_sfull(X, c), (c >> 1) & 1, a.wait_ns, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tS = tS0 + (c & 1) * BN;
        const int lo = glo - j * BN, hi = ghi - j * BN;   // valid columns: [lo, hi) within [0, 64), same for every row
        float v[64];
        tmem_ld64(tS, v);
        tmem_wait_ld();
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (lo <= 0 && hi >= BN) {
#pragma unroll
          for (int i = 0; i < 64; i += 8)
#pragma unroll
            for (int u = 0; u < 4; ++u) mx[u] = fmax3(mx[u], v[i + 2 * u], v[i + 2 * u + 1]);
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            v[i] = (i >= lo && i < hi) ? v[i] : -INFINITY;
            mx[i & 3] = fmaxf(mx[i & 3], v[i]);
          }
        }
        const float cm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
        const bool up = cm > m_run + C::kRaise;   // the group's first tile of the item: always (m_run = -inf)
        if (__any_sync(0xffffffffu, up)) {
          const float alpha = up ? ex2_approx(m_run - cm) : 1.f;
          l_run *= alpha;
          if (j > j0) {
            // O holds this group's earlier tiles of the item once the previous
            // P.V has completed (the ones before it completed before this S)
            if (!mbar_wait_warp(b_pv(X, c - 1), ((c - 1) >> 1) & 1, a.wait_ns, abort_flag)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
              float o[32];
              tmem_ld32(tO + cc * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] *= alpha;
              tmem_st32(tO + cc * 32, o);
            }
          }
          if (up) m_run = cm;
        }
        // pairs of columns through the packed two-lane fp32 instructions
        const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-m_run, -m_run);
        float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 x = __ffma2_rn(make_float2(v[2 * i], v[2 * i + 1]), sc2, nm2);
          v[2 * i] = ex2_approx(x.x);   // masked columns: 2^-inf = 0
          v[2 * i + 1] = ex2_approx(x.y);
          rs2[i & 1] = __fadd2_rn(rs2[i & 1], make_float2(v[2 * i], v[2 * i + 1]));
        }
        l_run += (rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y);
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
        tmem_st32u(tS, pk);
        const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 hv = make_float2(__uint_as_float(pk[i] << 16), __uint_as_float(pk[i] & 0xFFFF0000u));
          const float2 lv = __ffma2_rn(hv, neg1, make_float2(v[2 * i], v[2 * i + 1]));   // exact v - hi
          pk[i] = pack_bf16x2(lv.x, lv.y);
        }
        tmem_st32u(tS + 32, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(b_p(X, c));
      }
      if (!ok) break;
      // the epilogue input of the first chunk is in flight while the last P.V runs
      float4 ein[EC / 4];
      if (q >= 0 && has_res) load_in(row, 0, ein);
      // O is final once this item's last two P.V of the group have completed
      // (the earlier ones completed before the last S this group has seen)
      for (int t = (j1 - j0 >= 2 ? c - 2 : c - 1); t < c && ok; ++t)
        if (!mbar_wait_warp(b_pv(X, t), (t >> 1) & 1, a.wait_ns, abort_flag)) ok = false;
      if (!ok) break;
      // ------------------------------------------------------------------ epilogue
      tc_fence_after();
      const float inv_l = 1.f / l_run;
#pragma unroll 1
      for (int cc = 0; cc < D / EC; ++cc) {
        float4 enx[EC / 4];   // next chunk's input in flight while this chunk is finished
        if (q >= 0 && has_res && cc + 1 < D / EC) load_in(row, cc + 1, enx);
        float o[EC];
        tmem_ld16(tO + cc * EC, o);
        tmem_wait_ld();
        if (q >= 0) {
#pragma unroll
          for (int i = 0; i < EC; ++i) o[i] *= inv_l;
          if (MODE == kModeStep) {
            if (ep16 != nullptr) {
#pragma unroll
              for (int u = 0; u < EC / 8; ++u) {
                const uint32_t wv[4] = {__float_as_uint(ein[u].x), __float_as_uint(ein[u].y),
                                        __float_as_uint(ein[u].z), __float_as_uint(ein[u].w)};
#pragma unroll
                for (int e = 0; e < 4; ++e) {   // element 2e in the low half, 2e + 1 in the high half
                  o[8 * u + 2 * e] += __uint_as_float(wv[e] << 16);
                  o[8 * u + 2 * e + 1] += __uint_as_float(wv[e] & 0xFFFF0000u);
                }
              }
            } else if (has_res) {
#pragma unroll
              for (int u = 0; u < EC / 4; ++u) {
                o[4 * u + 0] += ein[u].x;
                o[4 * u + 1] += ein[u].y;
                o[4 * u + 2] += ein[u].z;
                o[4 * u + 3] += ein[u].w;
              }
            }
            uint4 *op = reinterpret_cast<uint4 *>(a.O + row + cc * EC);
#pragma unroll
            for (int u = 0; u < EC / 8; ++u) {
              uint4 wv;
              wv.x = pack_bf16x2(o[8 * u + 0], o[8 * u + 1]);
              wv.y = pack_bf16x2(o[8 * u + 2], o[8 * u + 3]);
              wv.z = pack_bf16x2(o[8 * u + 4], o[8 * u + 5]);
              wv.w = pack_bf16x2(o[8 * u + 6], o[8 * u + 7]);
              op[u] = wv;
            }
          } else {
            float4 *rp = reinterpret_cast<float4 *>(a.R_out + row + cc * EC);
#pragma unroll
            for (int u = 0; u < EC / 4; ++u)
              rp[u] = make_float4(ein[u].x - o[4 * u], ein[u].y - o[4 * u + 1], ein[u].z - o[4 * u + 2],
                                  ein[u].w - o[4 * u + 3]);
          }
        }
        if (cc + 1 < D / EC) {
#pragma unroll
          for (int u = 0; u < EC / 4; ++u) ein[u] = enx[u];
        }
        __syncwarp();   // the next TMEM load is warp-collective
      }
    }
    if (!ok && lane == 0 && !*abort_flag) {
      *abort_flag = 1;
      record_status(a.status, kStatusTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Union lists of group pairs, derived once per plan from kv_idx.
// One CTA of kPairThreads per (head, pair).  Output for pair p of head bh:
//   positions [0, k - s)        keys only group 2p keeps
//   positions [k - s, k)        keys both groups keep (s of them)
//   positions [k, 2k - s)       keys only group 2p+1 keeps
// and pair_len = 2k - s (k alone when group 2p+1 does not exist).  Within each
// segment keys stay in ascending order, so the lists are deterministic.
// Membership is found by binary search in the other group's ascending list.
// ---------------------------------------------------------------------------
constexpr int kPairThreads = 256;

__device__ __forceinline__ bool sorted_contains(const int32_t *L, int n, int x) {
  int lo = 0, hi = n;   // search [lo, hi)
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const int v = L[mid];
    if (v == x) return true;
    if (v < x) lo = mid + 1;
    else hi = mid;
  }
  return false;
}

// exclusive prefix count of `flag` over the CTA (in thread order) and the total
__device__ __forceinline__ int cta_exclusive_count(bool flag, int *warp_tot, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned m = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(m & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[warp] = __popc(m);
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kPairThreads / 32; ++w) {
    const int t = warp_tot[w];
    before += w < warp ? t : 0;
    all += t;
  }
  __syncthreads();   // warp_tot is reused by the next call
  *total = all;
  return before + in_warp;
}

__global__ void __launch_bounds__(kPairThreads) pair_build_kernel(const int32_t *kv_idx, int n_groups, int kk,
                                                                  int n_pairs, int32_t *pair_idx,
                                                                  int32_t *pair_len) {
  __shared__ int warp_tot[kPairThreads / 32];
  const int p = blockIdx.x, bh = blockIdx.y;
  const int32_t *A = kv_idx + (static_cast<size_t>(bh) * n_groups + 2 * p) * kk;
  int32_t *out = pair_idx + (static_cast<size_t>(bh) * n_pairs + p) * (2 * static_cast<size_t>(kk));
  const bool hasB = 2 * p + 1 < n_groups;
  if (!hasB) {
    for (int i = threadIdx.x; i < kk; i += kPairThreads) out[i] = A[i];
    if (threadIdx.x == 0) pair_len[static_cast<size_t>(bh) * n_pairs + p] = kk;
    return;
  }
  const int32_t *B = A + kk;
  // pass 1 over A: how many keys both keep (s), to place the shared segment
  int shared_cnt = 0;
  for (int base = 0; base < kk; base += kPairThreads) {
    const int i = base + static_cast<int>(threadIdx.x);
    const bool f = i < kk && sorted_contains(B, kk, A[i]);
    int tot;
    cta_exclusive_count(f, warp_tot, &tot);
    shared_cnt += tot;
  }
  // pass 2 over A: A-only keys from position 0, shared keys from k - s, in order
  int a_only = 0, both = 0;
  for (int base = 0; base < kk; base += kPairThreads) {
    const int i = base + static_cast<int>(threadIdx.x);
    const int x = i < kk ? A[i] : 0;
    const bool f = i < kk && sorted_contains(B, kk, x);
    int tot_f, tot_n;
    const int rf = cta_exclusive_count(f, warp_tot, &tot_f);
    const int rn = cta_exclusive_count(i < kk && !f, warp_tot, &tot_n);
    if (i < kk) out[f ? (kk - shared_cnt) + both + rf : a_only + rn] = x;
    both += tot_f;
    a_only += tot_n;
  }
  // pass over B: B-only keys from position k, in order
  int b_only = 0;
  for (int base = 0; base < kk; base += kPairThreads) {
    const int i = base + static_cast<int>(threadIdx.x);
    const int x = i < kk ? B[i] : 0;
    const bool nf = i < kk && !sorted_contains(A, kk, x);
    int tot;
    const int rn = cta_exclusive_count(nf, warp_tot, &tot);
    if (nf) out[kk + b_only + rn] = x;
    b_only += tot;
  }
  if (threadIdx.x == 0) pair_len[static_cast<size_t>(bh) * n_pairs + p] = kk + b_only;
}

}  // namespace mcs
