// attn_dual_kernel.cuh -- dense attention with two softmax warpgroups that
// take alternate key tiles.
//
// Used for the two dense modes of attn_kernel.cuh:
//  kModeDense     O = softmax(scale Q K^T) V over all N keys, bf16 out (the
//                 dense baseline, aiqbench.com abstract: "relative to dense
//                 attention");
//  kModePlanDense the dense pass of the plan: exact row statistics (m, l)
//                 over all keys plus the dense output in fp32, with P split
//                 into bf16 hi + lo parts and two P.V MMAs (~2^-17 relative
//                 error instead of 2^-9).
//
// CTA = 128 query rows x all key tiles of 128 keys:
//   warps 0-3  softmax warpgroup 0: key tiles 0, 2, 4, ...  (S0, O0)
//   warps 4-7  softmax warpgroup 1: key tiles 1, 3, 5, ...  (S1, O1)
//              thread t of either group owns query row t % 128 (TMEM lane)
//   warp  8    TMEM allocation and the single UMMA-issuing thread
//   warp  9    Q tile and the K ring, warp 10 the V ring (TMA 3D tile loads;
//              rows past the head's end load as zeros)
// Each group runs its own online softmax (row max m_g, sum l_g, output
// accumulator O_g in TMEM); the two are merged once, in the epilogue:
//   m = max(m0, m1),  l = l0 2^(m0-m) + l1 2^(m1-m),
//   O = (O0 2^(m0-m) + O1 2^(m1-m)) / l.
// The two groups work on different tiles at the same time, so one group's
// TMEM loads and stores, and its wait for the next S, overlap the other's
// exponentials.  The tensor pipe runs QK(0) QK(1), then per key tile j:
// PV(j) into O_(j%2), QK(j+2) into S_(j%2).  Because QK(j) is issued after
// PV(j-2), a group that sees S of tile j ready also knows that its O holds
// every earlier tile of its own, and nothing writes that O until it
// publishes P of tile j: it can rescale O with no further wait.
// S is read in two 64-column chunks.  P of chunk c goes over the chunk's own
// columns [64c, 64c+64) of S: bf16 hi pairs in the first 32, lo pairs (plan
// mode) in the last 32.  The exponentials of a chunk use the group's running
// max from before the chunk; only when a row's chunk max exceeds it by more
// than 2^kRaise (log2 units: always on the group's first chunk, else rare)
// are m, l, O and any P already written for the tile rescaled.
// TMEM: S0, S1 (128 columns each), O0, O1 (D columns each).
// Every wait is bounded.
#pragma once

#include "attn_kernel.cuh"

namespace mcs {

template <int D, int MODE>
struct DualCfg {
  static_assert(MODE == kModeDense || MODE == kModePlanDense, "dense modes only");
  static constexpr int BM = 128, BN = 128;
  static constexpr bool kSplit = (MODE == kModePlanDense);
  static constexpr int NK = D == 64 ? 6 : 3;   // K ring depth
  static constexpr int NV = D == 64 ? 6 : 3;   // V ring depth
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NV * KV_BYTES;
  static constexpr int N_BAR = 1 + 2 * NK + 2 * NV + 7;   // q, k/v full/empty, s_full[2], p[2], pv[2], drain
  static constexpr int OFF_XCH = OFF_BAR + 8 * N_BAR;      // 128 x float2: the epilogue's merge
  static constexpr int OFF_MISC = OFF_XCH + 128 * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;          // + slack to align the base to 1 KB
  static constexpr int MMA_WARP = 8, KQ_WARP = 9, V_WARP = 10;
  static constexpr int THREADS = 11 * 32;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
  static constexpr float kRaise = 32.f;   // lazy rescale bound, as in attn_kernel.cuh
};

template <int D, int MODE>
__global__ void __launch_bounds__(DualCfg<D, MODE>::THREADS, 1) attn_dual_kernel(const __grid_constant__ AttnArgs a) {
  using C = DualCfg<D, MODE>;
  constexpr int BM = C::BM, BN = C::BN, NK = C::NK, NV = C::NV;
  constexpr int NDB = D / 64;                       // 64-column (128-byte) blocks per row
  constexpr uint32_t TILE_TX = 128u * D * 2u;       // bytes of one 128-row tile
  constexpr int OCOLS = D / 2;                      // output columns per thread in the epilogue

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
  // one barrier of each kind per softmax group (= per key-tile parity)
  const uint32_t bx = bar0 + 8 * (1 + 2 * NK + 2 * NV);
  auto b_sfull = [&](int j) { return bx + 8 * (j & 1); };
  auto b_p = [&](int j) { return bx + 16 + 8 * (j & 1); };
  auto b_pv = [&](int j) { return bx + 32 + 8 * (j & 1); };
  const uint32_t b_drain = bx + 48;
  float2 *xch = reinterpret_cast<float2 *>(smem + C::OFF_XCH);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int N = a.N;
  const int per_head = (N + BM - 1) / BM;
  const int tile = blockIdx.x % per_head;   // one CTA per (head, query tile), head-major
  const int bh = blockIdx.x / per_head;
  const size_t head = static_cast<size_t>(bh) * N;
  const int T = (N + BN - 1) / BN;

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
    for (int g = 0; g < 2; ++g) {
      mbar_init(b_sfull(g), 1);
      mbar_init(b_p(g), 128);
      mbar_init(b_pv(g), 1);
    }
    mbar_init(b_drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::KQ_WARP && lane == 0) {
    tma_prefetch_desc(&a.tmQ);
    tma_prefetch_desc(&a.tmK);
    tma_prefetch_desc(&a.tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == C::KQ_WARP || warp == C::V_WARP) {
    // ------------------------------------------------------------------ TMA producers
    if (lane == 0) {
      const bool is_k = warp == C::KQ_WARP;
      const void *tm = is_k ? static_cast<const void *>(&a.tmK) : static_cast<const void *>(&a.tmV);
      const int NS = is_k ? NK : NV;
      const uint32_t ring = is_k ? sK0 : sV0;
      if (is_k) {
        mbar_arrive_expect_tx(b_q, TILE_TX);
#pragma unroll
        for (int db = 0; db < NDB; ++db) tma_load_3d(sQ + db * (BM * 128), &a.tmQ, db * 64, tile * BM, bh, b_q);
      }
      bool ok = true;
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        const int s = j % NS;
        if (!mbar_wait(is_k ? b_kempty(s) : b_vempty(s), ((j / NS) & 1) ^ 1, a.wait_ns, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t full = is_k ? b_kfull(s) : b_vfull(s);
        mbar_arrive_expect_tx(full, TILE_TX);
#pragma unroll
        for (int db = 0; db < NDB; ++db)
          tma_load_3d(ring + s * C::KV_BYTES + db * (BN * 128), tm, db * 64, j * BN, bh, full);
        ++issued;
      }
      if (!ok && !*abort_flag) {
        *abort_flag = 1;
        record_status(a.status, kStatusTimeout);
      }
      // never leave the CTA with a copy still landing in its shared memory
      volatile int never = 0;
      for (int t = (issued > NS ? issued - NS : 0); t < issued; ++t)
        mbar_wait(is_k ? b_kfull(t % NS) : b_vfull(t % NS), (t / NS) & 1, 2000000000ull, &never);
      if (is_k) mbar_wait(b_q, 0, 2000000000ull, &never);
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------------ UMMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, 1);
      bool ok = mbar_wait(b_q, 0, a.wait_ns, abort_flag);
      auto issue_qk = [&](int j) -> bool {
        const int s = j % NK;
        if (!mbar_wait(b_kfull(s), (j / NK) & 1, a.wait_ns, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kb = sK0 + s * C::KV_BYTES;
        const uint32_t tS = tbase + ((j & 1) ? C::COL_S1 : C::COL_S0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          umma_bf16_ss(tS, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), idesc_qk,
                       kk > 0 ? 1u : 0u);
        }
        umma_commit(b_sfull(j));
        umma_commit(b_kempty(s));
        return true;
      };
      // P of keys 64c .. 64c+63 sits at columns 64c + [0, 32) (hi pairs) and
      // 64c + [32, 64) (lo pairs) of its S buffer
      auto issue_pv = [&](int j) -> bool {
        const int s = j % NV;
        if (!mbar_wait(b_p(j), (j >> 1) & 1, a.wait_ns, abort_flag)) return false;
        if (!mbar_wait(b_vfull(s), (j / NV) & 1, a.wait_ns, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vb = sV0 + s * C::KV_BYTES;
        const uint32_t tP = tbase + ((j & 1) ? C::COL_S1 : C::COL_S0);
        const uint32_t tO = tbase + ((j & 1) ? C::COL_O1 : C::COL_O0);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t acol = 64 * (kk >> 2) + 8 * (kk & 3);
          const uint64_t bdesc = sdesc_sw128(vb + kk * 16 * 128, BN * 128, 1024);
          umma_bf16_ts(tO, tP + acol, bdesc, idesc_pv, (j >= 2 || kk > 0) ? 1u : 0u);
        }
        if (C::kSplit) {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint32_t acol = 64 * (kk >> 2) + 32 + 8 * (kk & 3);
            const uint64_t bdesc = sdesc_sw128(vb + kk * 16 * 128, BN * 128, 1024);
            umma_bf16_ts(tO, tP + acol, bdesc, idesc_pv, 1u);
          }
        }
        umma_commit(b_pv(j));
        umma_commit(b_vempty(s));
        return true;
      };
      if (ok) ok = issue_qk(0);
      if (ok && T > 1) ok = issue_qk(1);
      for (int j = 0; j < T && ok; ++j) {
        ok = issue_pv(j);
        if (ok && j + 2 < T) ok = issue_qk(j + 2);
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
    // ------------------------------------------------------------------ softmax groups (warps 0-7)
    const int grp = warp >> 2;
    const int r = (warp & 3) * 32 + lane;            // row == TMEM lane
    const int qrow = tile * BM + r;
    const int q = qrow < N ? qrow : -1;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + lane_addr + (grp ? C::COL_S1 : C::COL_S0);
    const uint32_t tOg = tbase + lane_addr + (grp ? C::COL_O1 : C::COL_O0);
    const float sl2 = a.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int j_last = -1;
    for (int j = grp; j < T; j += 2) {
      if (!mbar_wait_warp(b_sfull(j), (j >> 1) & 1, a.wait_ns, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float rs = 0.f;   // this tile's sum, relative to m_run
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float v[64];
        tmem_ld64(tS + 64 * c, v);
        tmem_wait_ld();
        const int nvalid = N - j * BN - 64 * c;   // valid columns of the chunk (may be <= 0)
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (nvalid >= 64) {
#pragma unroll
          for (int i = 0; i < 64; i += 8)
#pragma unroll
            for (int u = 0; u < 4; ++u) mx[u] = fmax3(mx[u], v[i + 2 * u], v[i + 2 * u + 1]);
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            v[i] = i < nvalid ? v[i] : -INFINITY;
            mx[i & 3] = fmaxf(mx[i & 3], v[i]);
          }
        }
        const float cm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
        const bool up = cm > m_run + C::kRaise;   // first chunk of the group: always (m_run = -inf)
        if (__any_sync(0xffffffffu, up)) {
          // the row max moved: rescale what this group holds for the row
          // (after this thread's earlier TMEM stores have landed)
          tmem_wait_st();
          const float alpha = up ? ex2_approx(m_run - cm) : 1.f;
          l_run *= alpha;
          rs *= alpha;
          if (c == 1) {   // P of chunk 0 of this tile, already in TMEM
            if (C::kSplit) {
              float p[64];
              tmem_ld64(tS, p);
              tmem_wait_ld();
              uint32_t hi[32], lo[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const uint32_t h = __float_as_uint(p[i]), l = __float_as_uint(p[32 + i]);
                const float x0 = (__uint_as_float(h << 16) + __uint_as_float(l << 16)) * alpha;
                const float x1 = (__uint_as_float(h & 0xFFFF0000u) + __uint_as_float(l & 0xFFFF0000u)) * alpha;
                const uint32_t nh = pack_bf16x2(x0, x1);
                const uint32_t nl = pack_bf16x2(x0 - __uint_as_float(nh << 16), x1 - __uint_as_float(nh & 0xFFFF0000u));
                hi[i] = up ? nh : h;
                lo[i] = up ? nl : l;
              }
              tmem_st32u(tS, hi);
              tmem_st32u(tS + 32, lo);
            } else {
              float p[32];
              tmem_ld32(tS, p);
              tmem_wait_ld();
              uint32_t hi[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const uint32_t h = __float_as_uint(p[i]);
                const uint32_t nh = pack_bf16x2(__uint_as_float(h << 16) * alpha, __uint_as_float(h & 0xFFFF0000u) * alpha);
                hi[i] = up ? nh : h;
              }
              tmem_st32u(tS, hi);
            }
          }
          if (j >= 2) {   // O_g holds this group's earlier tiles, all complete (see above)
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
              float o[32];
              tmem_ld32(tOg + cc * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] *= alpha;
              tmem_st32(tOg + cc * 32, o);
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
        rs += (rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y);
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
        tmem_st32u(tS + 64 * c, pk);
        if (C::kSplit) {
          const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 h = make_float2(__uint_as_float(pk[i] << 16), __uint_as_float(pk[i] & 0xFFFF0000u));
            const float2 lo = __ffma2_rn(h, neg1, make_float2(v[2 * i], v[2 * i + 1]));   // exact v - h
            pk[i] = pack_bf16x2(lo.x, lo.y);
          }
          tmem_st32u(tS + 64 * c + 32, pk);
        }
      }
      l_run += rs;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(b_p(j));
      j_last = j;
    }
    // this group's O is final once its last P.V has completed (its earlier
    // ones completed before the last Q.K^T it has seen)
    if (ok && j_last >= 0 && !mbar_wait_warp(b_pv(j_last), (j_last >> 1) & 1, a.wait_ns, abort_flag)) ok = false;
    if (!ok && lane == 0 && !*abort_flag) {
      *abort_flag = 1;
      record_status(a.status, kStatusTimeout);
    }
    // ------------------------------------------------------------------ merge + epilogue
    // group 1 posts (m1, l1); group 0 merges and posts the two O factors.
    // Both groups pass both barriers whatever happened above.
    if (grp == 1) xch[r] = make_float2(m_run, l_run);
    asm volatile("bar.sync 1, 256;" ::: "memory");
    float f0, f1, m_fin = 0.f, l_fin = 0.f;
    if (grp == 0) {
      const float2 g1 = xch[r];
      m_fin = fmaxf(m_run, g1.x);
      const float a0 = ex2_approx(m_run - m_fin);
      const float a1 = T >= 2 ? ex2_approx(g1.x - m_fin) : 0.f;
      l_fin = l_run * a0 + g1.y * a1;
      const float inv_l = 1.f / l_fin;
      f0 = a0 * inv_l;
      f1 = a1 * inv_l;
      xch[r] = make_float2(f0, f1);
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (grp == 1) {
      const float2 f = xch[r];
      f0 = f.x;
      f1 = f.y;
    }
    if (ok) {
      tc_fence_after();
      const uint32_t tO0 = tbase + lane_addr + C::COL_O0 + grp * OCOLS;
      const uint32_t tO1 = tbase + lane_addr + C::COL_O1 + grp * OCOLS;
      const size_t row = (head + (q >= 0 ? q : 0)) * D + grp * OCOLS;
#pragma unroll 1
      for (int cc = 0; cc < OCOLS / 32; ++cc) {
        float o[32], o1[32];
        tmem_ld32(tO0 + cc * 32, o);
        if (T >= 2) tmem_ld32(tO1 + cc * 32, o1);   // O1 is never written when there is one key tile
        tmem_wait_ld();
        if (q >= 0) {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = T >= 2 ? fmaf(o[i], f0, o1[i] * f1) : o[i] * f0;
          if (MODE == kModePlanDense) {
            float4 *op = reinterpret_cast<float4 *>(a.O32 + row + cc * 32);
#pragma unroll
            for (int u = 0; u < 8; ++u) op[u] = make_float4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
          }
          if (MODE == kModeDense || a.O != nullptr) {
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
        }
        __syncwarp();   // the next TMEM load is warp-collective
      }
      if (MODE == kModePlanDense && q >= 0 && grp == 0) {
        a.row_m[head + q] = m_fin;
        a.row_l[head + q] = l_fin;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace mcs
