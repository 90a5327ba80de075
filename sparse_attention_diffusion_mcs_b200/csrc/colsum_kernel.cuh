// colsum_kernel.cuh -- group probability sums, step a3 of the plan.
//
//   colsum[g, j] = sum_{i in group g} P_ij,  P_ij = 2^(s_ij*scale*log2e - m_i) / l_i
//                                                = 2^(s_ij*scale*log2e - c_i),  c_i = m_i + log2(l_i)
//
// with (m_i, l_i) the exact row statistics from the dense pass ("KV indices
// selected using exact attention probabilities", aiqbench.com abstract; the
// per-group sum is the selection score this library adopts).
//
// The score tile is computed transposed, S^T = K_tile . Q_g^T (keys on TMEM
// lanes, the group's queries on columns), so each thread owns one key and the
// sum over the group is a private loop over its TMEM row: no cross-thread
// reduction.  CTA = one (head, group); loops over all N/128 key tiles.
//   warps 0-3 reduce, warp 4 issues UMMA, warp 5 loads the group's queries
//   (TMA tile::gather4) and streams K tiles (TMA 3D tiles), warp 6 idles.
// Two CTAs share an SM (256 TMEM columns and < 114 KB of shared memory each),
// so each SM sub-partition has two reducing warps to hide TMEM and MUFU
// latency.  The reducers keep the next 32-column chunk's TMEM load in flight,
// and compute a quarter of the exponentials on the FMA pipe (ex2_fma) so that
// the MUFU pipe, which bounds this kernel, carries three quarters.
#pragma once

#include "mcs_common.cuh"

namespace mcs {

struct alignas(64) ColsumArgs {
  CUtensorMap tmQ;          // gather map over [BH*N, D]
  CUtensorMap tmK;          // tile map over [BH, N, D]
  const int32_t *perm;      // [BH, N]
  const float *row_m;       // [BH, N] (log2 domain)
  const float *row_l;       // [BH, N]
  float *colsum;            // [BH, n_groups, N]
  int N, G, n_groups;
  float scale_log2;
  unsigned *status;
  uint64_t wait_ns;
};

// which of every 8 consecutive exponentials run on the FMA pipe (bit i: column
// i mod 8); the rest use the MUFU ex2
#ifndef MCS_COLSUM_FMA_EXP_MASK
#define MCS_COLSUM_FMA_EXP_MASK 0x88u
#endif
constexpr unsigned kFmaExpMask = MCS_COLSUM_FMA_EXP_MASK;

template <int D>
struct ColsumCfg {
  static constexpr int BM = 128, BN = 128;   // BM keys per tile (MMA M), BN queries (MMA N)
  static constexpr int NST = D == 64 ? 4 : 2;   // K ring depth (two CTAs per SM)
  static constexpr int Q_BYTES = BN * D * 2;
  static constexpr int K_BYTES = BM * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_STAT = OFF_K + NST * K_BYTES;     // c_i = m_i + log2(l_i), 128 floats
  static constexpr int OFF_BAR = OFF_STAT + 128 * 8;
  static constexpr int N_BAR = 1 + 2 * NST + 5;              // q, k full/empty, s_full[2], s_free[2], drain
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BAR;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 256;
};

template <int D>
__global__ void __launch_bounds__(224, 2) colsum_kernel(const __grid_constant__ ColsumArgs a) {
  using C = ColsumCfg<D>;
  constexpr int BM = C::BM, NST = C::NST;
  constexpr int NDB = D / 64;
  constexpr uint32_t TILE_TX = 128u * D * 2u;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sK0 = sbase + C::OFF_K;
  float *stat = reinterpret_cast<float *>(smem + C::OFF_STAT);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t b_q = bar0;
  auto b_kfull = [&](int s) { return bar0 + 8 * (1 + s); };
  auto b_kempty = [&](int s) { return bar0 + 8 * (1 + NST + s); };
  const uint32_t b_sfull0 = bar0 + 8 * (1 + 2 * NST);
  const uint32_t b_sfree0 = bar0 + 8 * (3 + 2 * NST);
  const uint32_t b_drain = bar0 + 8 * (5 + 2 * NST);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int g = blockIdx.x;
  const int bh = blockIdx.y;
  const int N = a.N;
  const size_t head = static_cast<size_t>(bh) * N;
  const int T = (N + BM - 1) / BM;

  auto q_token = [&](int r) -> int {
    const int gr = g * a.G + r;
    if (r >= a.G || gr >= N) return -1;
    const int q = a.perm[head + gr];
    if (static_cast<unsigned>(q) >= static_cast<unsigned>(N)) {   // corrupt metadata: never gather out of range
      record_status(a.status, kStatusBadMeta);
      return -1;
    }
    return q;
  };

  if (tid == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(b_kfull(s), 1);
      mbar_init(b_kempty(s), 1);
    }
    mbar_init(b_sfull0, 1);
    mbar_init(b_sfull0 + 8, 1);
    mbar_init(b_sfree0, 128);
    mbar_init(b_sfree0 + 8, 128);
    mbar_init(b_drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (tid < 128) {
    const int q = q_token(tid);
    // fold the normaliser into the exponent (stored negated, the addend of
    // the scale-and-shift); a padding query contributes 2^-inf = 0
    stat[tid] = q >= 0 ? -(a.row_m[head + q] + log2f(a.row_l[head + q])) : -INFINITY;
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 5) {
    const int lane = tid & 31;
    {
      int rows[4];
      const int q0 = q_token(0);
      const int fallback = q0 >= 0 ? q0 : 0;   // padding queries re-read a valid row (their stats zero them)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q = q_token(4 * lane + i);
        rows[i] = static_cast<int>(head) + (q >= 0 ? q : fallback);
      }
      if (lane == 0) mbar_arrive_expect_tx(b_q, TILE_TX);
      __syncwarp();
#pragma unroll
      for (int db = 0; db < NDB; ++db)
        tma_gather4(sQ + db * (128 * 128) + lane * 512, &a.tmQ, db * 64, rows[0], rows[1], rows[2], rows[3], b_q);
    }
    bool ok = true;
    int issued = 0;
    if (lane == 0) {
      for (int j = 0; j < T; ++j) {
        const int s = j % NST;
        if (!mbar_wait(b_kempty(s), ((j / NST) & 1) ^ 1, a.wait_ns, abort_flag)) { ok = false; break; }
        const uint32_t dK = sK0 + s * C::K_BYTES;
        mbar_arrive_expect_tx(b_kfull(s), TILE_TX);
#pragma unroll
        for (int db = 0; db < NDB; ++db) tma_load_3d(dK + db * (BM * 128), &a.tmK, db * 64, j * BM, bh, b_kfull(s));
        ++issued;
      }
      if (!ok && !*abort_flag) {
        *abort_flag = 1;
        record_status(a.status, kStatusTimeout);
      }
      // never leave the CTA with a copy still landing in its shared memory
      volatile int never = 0;
      for (int t = (issued > NST ? issued - NST : 0); t < issued; ++t)
        mbar_wait(b_kfull(t % NST), (t / NST) & 1, 2000000000ull, &never);
      mbar_wait(b_q, 0, 2000000000ull, &never);
    }
    __syncwarp();
  } else if (warp == 4) {
    if (tid == 128) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, 128, 0);
      bool ok = mbar_wait(b_q, 0, a.wait_ns, abort_flag);
      for (int j = 0; j < T && ok; ++j) {
        const int s = j % NST;
        const int b = j & 1;
        if (j >= 2 && !mbar_wait(b_sfree0 + 8 * b, ((j >> 1) - 1) & 1, a.wait_ns, abort_flag)) {
          ok = false;
          break;
        }
        if (!mbar_wait(b_kfull(s), (j / NST) & 1, a.wait_ns, abort_flag)) { ok = false; break; }
        tc_fence_after();
        fence_proxy_async_smem();
        const uint32_t kb = sK0 + s * C::K_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          umma_bf16_ss(tbase + b * 128, sdesc_sw128(kb + off, 16, 1024),
                       sdesc_sw128(sQ + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(b_sfull0 + 8 * b);
        umma_commit(b_kempty(s));
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
  } else if (warp < 4) {
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    float *out = a.colsum + (static_cast<size_t>(bh) * a.n_groups + g) * N;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int b = j & 1;
      if (!mbar_wait_warp(b_sfull0 + 8 * b, (j >> 1) & 1, a.wait_ns, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float2 acc01 = make_float2(0.f, 0.f), acc23 = make_float2(0.f, 0.f);
      const float2 sc2 = make_float2(sl2, sl2);
      float v[2][32];
      tmem_ld32(tbase + lane_addr + b * 128, v[0]);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float (&cur)[32] = v[cc & 1];
        tmem_wait_ld();
        if (cc + 1 < 4) tmem_ld32(tbase + lane_addr + b * 128 + (cc + 1) * 32, v[(cc + 1) & 1]);
        const float4 *c4 = reinterpret_cast<const float4 *>(stat + cc * 32);
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 c = c4[i / 4];     // same address in every lane: one broadcast read
          // two queries per packed two-lane fp32 instruction
          const float2 x01 = __ffma2_rn(make_float2(cur[i], cur[i + 1]), sc2, make_float2(c.x, c.y));
          const float2 x23 = __ffma2_rn(make_float2(cur[i + 2], cur[i + 3]), sc2, make_float2(c.z, c.w));
          const float x[4] = {x01.x, x01.y, x23.x, x23.y};
          float e[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) e[u] = ((kFmaExpMask >> ((i + u) & 7)) & 1u) ? ex2_fma(x[u]) : ex2_approx(x[u]);
          acc01 = __fadd2_rn(acc01, make_float2(e[0], e[1]));
          acc23 = __fadd2_rn(acc23, make_float2(e[2], e[3]));
        }
      }
      const float acc0 = acc01.x + acc01.y, acc2 = acc23.x + acc23.y;
      tc_fence_before();
      mbar_arrive(b_sfree0 + 8 * b);
      const int key = j * BM + tid;
      if (key < N) out[key] = acc0 + acc2;
    }
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
