// micro_pipes.cu -- libmcs_micro.so, second part: the two execution rates
// the reused step's roofline rests on, each measured on its own
// (include/mcs_micro.h): the MUFU exponential rate per SM, and the tcgen05
// MMA rate of the step's two MMA shapes, alone and while other warps of the
// same SM keep the MUFU or FMA pipe busy, as the softmax does.  Measurement
// only.
#include <cstring>

#include "../../include/mcs_micro.h"
#include "mcs_common.cuh"

using namespace mcs;

namespace {

// ---------------------------------------------------------------- exponentials
// Each thread runs 8 independent chains v = 2^v - 1.5 (fixed point -1: the
// values stay finite), `iters` steps each; cycles of the whole CTA by clock64.
__global__ void micro_ex2_kernel(int iters, unsigned long long *out) {
  __shared__ unsigned long long t_begin, t_end;
  float v[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) v[c] = -1.f + 0.001f * c;
  __syncthreads();
  if (threadIdx.x == 0) t_begin = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int c = 0; c < 8; ++c) v[c] = ex2_approx(v[c]) - 1.5f;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    t_end = clock64();
    out[blockIdx.x] = t_end - t_begin;
  }
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) s += v[c];
  if (s == 12345.f) out[gridDim.x + blockIdx.x] = 1;   // keeps the chains live
}

// ---------------------------------------------------------------- MMA rate
constexpr int kMmaThreads = 9 * 32;        // warp 0 issues MMAs, warps 1-8 load the other pipes
constexpr int A_BYTES = 128 * 128 * 2;     // 128 rows x 128 columns bf16, 128-byte swizzle, K-major
constexpr int B_BYTES = 128 * 128 * 2;
constexpr int OFF_BAR = A_BYTES + B_BYTES;
// more shared memory than two CTAs could share, so each SM runs one CTA (and
// one TMEM allocation) at a time
constexpr int MMA_SMEM = 120 * 1024;
static_assert(OFF_BAR + 64 + 1024 <= MMA_SMEM, "operands and barriers fit");

// The issuing warp's loop, with the shape and the number of accumulators
// fixed at compile time and every descriptor formed before the timed loop,
// as in the step's MMA warp: nothing but the MMAs themselves between MMAs.
template <int SHAPE, int CHAINS>
__device__ __forceinline__ void issue_mmas(uint32_t tbase, uint32_t sA, uint32_t sB, int batches) {
  constexpr int NB = SHAPE == 0 ? 64 : 128;                 // N, and the B operand's rows for SS
  constexpr uint32_t idesc = SHAPE == 1 ? idesc_bf16_f32(128, 128, 1) : idesc_bf16_f32(128, NB, 0);
  const uint64_t da = sdesc_sw128(sA, 16, 1024);
  const uint64_t db = SHAPE == 1 ? sdesc_sw128(sB, 128 * 128, 1024) : sdesc_sw128(sB, 16, 1024);
  uint64_t A[8], B[8];
  uint32_t At[8];
#pragma unroll
  for (int k16 = 0; k16 < 8; ++k16) {
    A[k16] = da + ((((k16 >> 2) * (128 * 128)) + (k16 & 3) * 32) >> 4);
    B[k16] = SHAPE == 1 ? db + ((k16 * 16 * 128) >> 4) : db + ((((k16 >> 2) * (NB * 128)) + (k16 & 3) * 32) >> 4);
    At[k16] = tbase + 256 + 8 * k16;
  }
  for (int b = 0; b < batches; ++b) {
#pragma unroll
    for (int k16 = 0; k16 < 8; ++k16) {
#pragma unroll
      for (int c = 0; c < CHAINS; ++c) {
        const uint32_t acc = (b > 0 || k16 > 0) ? 1u : 0u;
        const uint32_t d = tbase + c * NB;
        if constexpr (SHAPE == 1) umma_bf16_ts_elect(d, At[k16], B[k16], idesc, acc);
        else umma_bf16_ss_elect(d, A[k16], B[k16], idesc, acc);
      }
    }
  }
}

// shape 0: SS, M = 128, N = 64 (the step's Q.K^T); 1: TS, M = 128, N = 128,
// A from TMEM, B MN-major (the step's P.V); 2: SS, M = 128, N = 128.
template <int SHAPE, int CHAINS>
__global__ void __launch_bounds__(kMmaThreads, 1) micro_mma_kernel(int batches, int load, unsigned long long *out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const uint32_t sA = smem_u32(smem), sB = sA + A_BYTES;
  const uint32_t bar = sA + OFF_BAR;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 16);
  volatile int *done = reinterpret_cast<volatile int *>(smem + OFF_BAR + 32);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // finite operands: zeros in shared memory and in TMEM's A columns
  for (int i = threadIdx.x; i < (A_BYTES + B_BYTES) / 16; i += kMmaThreads)
    reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *done = 0;
    mbar_init_fence();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  if (warp >= 1 && warp <= 4) {   // warps 1-4 cover the four TMEM lane quadrants
    const uint32_t lanes = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float z[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) z[i] = 0.f;
    tmem_st32(tbase + lanes + 256, z);
    tmem_st32(tbase + lanes + 288, z);
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    const unsigned long long t0 = clock64();
    issue_mmas<SHAPE, CHAINS>(tbase, sA, sB, batches);
    umma_commit_elect(bar);
    volatile int never = 0;
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, 0, 2000000000ull, &never) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    const unsigned long long t1 = clock64();
    if (lane == 0) {
      out[3 * blockIdx.x + 0] = t1 - t0;
      out[3 * blockIdx.x + 1] = static_cast<unsigned long long>(batches) * 8 * CHAINS;
      out[3 * blockIdx.x + 2] = ok ? 0 : 1;
      *done = 1;
    }
    __syncwarp();
  } else if (load != 0) {
    // keep this SM's MUFU (load 1) or FMA (load 2) pipe busy until the MMAs are
    // done: 8 independent chains per thread; at most 2^22 rounds whatever happens
    float v[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) v[c] = -1.f + 0.001f * (c + threadIdx.x);
    if (load == 1) {
      for (int round = 0; round < (1 << 22) && !*done; ++round)
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 8; ++c) v[c] = ex2_approx(v[c]) - 1.5f;
    } else {
      for (int round = 0; round < (1 << 22) && !*done; ++round)
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 8; ++c) v[c] = fmaf(v[c], 0.5f, -0.5f);
    }
    float sum = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) sum += v[c];
    if (sum == 12345.f) out[3 * gridDim.x] = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <int SHAPE, int CHAINS>
cudaError_t launch_mma(int ctas, int batches, int load, unsigned long long *out, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(micro_mma_kernel<SHAPE, CHAINS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       MMA_SMEM);
  if (e != cudaSuccess) return e;
  micro_mma_kernel<SHAPE, CHAINS><<<ctas, kMmaThreads, MMA_SMEM, s>>>(batches, load, out);
  return cudaGetLastError();
}

}  // namespace

extern "C" {

mcs_status mcs_micro_ex2(int ctas, int warps, int iters, unsigned long long *cycles, mcs_stream_t stream) {
  if (!cycles || ctas < 1 || warps < 1 || warps > 32 || iters < 1) return MCS_ERR_INVALID_ARG;
  micro_ex2_kernel<<<ctas, warps * 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(iters, cycles);
  return cudaGetLastError() == cudaSuccess ? MCS_OK : MCS_ERR_CUDA;
}

mcs_status mcs_micro_mma(int ctas, int shape, int batches, int load, int chains, unsigned long long *out,
                         mcs_stream_t stream) {
  if (!out || ctas < 1 || shape < 0 || shape > 2 || batches < 1 || load < 0 || load > 2) return MCS_ERR_INVALID_ARG;
  // accumulators must stay clear of the TS operand's columns [256, 320)
  if (chains < 1 || chains > (shape == 0 ? 4 : 2)) return MCS_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (shape == 0)
    e = chains == 1 ? launch_mma<0, 1>(ctas, batches, load, out, s)
                    : (chains == 2 ? launch_mma<0, 2>(ctas, batches, load, out, s)
                                   : (chains == 3 ? launch_mma<0, 3>(ctas, batches, load, out, s)
                                                  : launch_mma<0, 4>(ctas, batches, load, out, s)));
  else if (shape == 1)
    e = chains == 1 ? launch_mma<1, 1>(ctas, batches, load, out, s) : launch_mma<1, 2>(ctas, batches, load, out, s);
  else
    e = chains == 1 ? launch_mma<2, 1>(ctas, batches, load, out, s) : launch_mma<2, 2>(ctas, batches, load, out, s);
  return e == cudaSuccess ? MCS_OK : MCS_ERR_CUDA;
}

}  // extern "C"
