// micro_gather.cu -- libmcs_micro.so: the index-listed row gather rate of one
// SM, measured on its own (include/mcs_micro.h).  Measurement only.
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "../../include/mcs_micro.h"
#include "mcs_common.cuh"

using namespace mcs;

namespace {

constexpr int NS = 4;                    // ring slots
constexpr int ROWS = 128;                // rows per tile
constexpr int TILE = ROWS * 256;         // bytes per tile (bf16 rows of 128)
constexpr int MAXW = 8;                  // producer warps at most
constexpr int THREADS = (MAXW + 1) * 32; // + one consumer warp
constexpr int SMEM = NS * TILE + 8 * 2 * NS + 16 + 1024;

struct alignas(64) MicroArgs {
  CUtensorMap tm_rows;   // 2D, box {64, 1}: gather4 source
  CUtensorMap tm_tile;   // 2D, box {64, 128}: contiguous tiles
  const bf16 *src;
  const int32_t *idx;
  size_t rows;
  int tiles, mode, warps;
  unsigned *status;
  uint64_t wait_ns;
};

__device__ unsigned g_micro_status;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// arrive on `bar` once this thread's earlier cp.async copies have landed
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__global__ void __launch_bounds__(THREADS, 1) micro_gather_kernel(const __grid_constant__ MicroArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const uint32_t ring = smem_u32(smem);
  const uint32_t bar0 = ring + NS * TILE;
  auto full = [&](int s) { return bar0 + 8 * s; };
  auto empty = [&](int s) { return bar0 + 8 * (NS + s); };
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + NS * TILE + 16 * NS);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int W = a.warps;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full(s), a.mode == MCS_MICRO_CP_ASYNC ? 32 * W : 1);
      mbar_init(empty(s), 1);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();
  const int32_t *my = a.idx + static_cast<size_t>(blockIdx.x) * a.tiles * ROWS;
  auto row_of = [&](int t, int r) -> int {
    int key = my[static_cast<size_t>(t) * ROWS + r];
    if (key < 0 || static_cast<size_t>(key) >= a.rows) {
      record_status(a.status, kStatusBadMeta);
      key = 0;
    }
    return key;
  };
  bool ok = true;
  if (warp == MAXW) {
    // consumer: free each slot as soon as it is full
    if (lane == 0) {
      for (int t = 0; t < a.tiles && ok; ++t)
        if ((ok = mbar_wait(full(t % NS), (t / NS) & 1, a.wait_ns, abort_flag))) mbar_arrive(empty(t % NS));
    }
  } else if (warp < W) {
    for (int t = 0; t < a.tiles && ok; ++t) {
      const int s = t % NS;
      int got = 1;
      if (lane == 0) got = mbar_wait(empty(s), ((t / NS) & 1) ^ 1, a.wait_ns, abort_flag);
      if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
      const uint32_t dst = ring + s * TILE;
      if (a.mode == MCS_MICRO_GATHER4) {
        if (warp == 0 && lane == 0) mbar_arrive_expect_tx(full(s), TILE);
        __syncwarp();
        // 64 operations per tile (32 row quads x 2 column blocks): op o -> warp o % W
        for (int o = warp + W * lane; o < 64; o += W * 32) {
          const int quad = o % 32, db = o / 32;
          tma_gather4(dst + db * (ROWS * 128) + quad * 512, &a.tm_rows, db * 64, row_of(t, 4 * quad),
                      row_of(t, 4 * quad + 1), row_of(t, 4 * quad + 2), row_of(t, 4 * quad + 3), full(s));
        }
      } else if (a.mode == MCS_MICRO_CP_ASYNC) {
        // 16 chunks of 16 bytes per row, stored in the same 128-byte-swizzled
        // layout the tensor-core tiles use
        for (int c = warp * 32 + lane; c < ROWS * 16; c += W * 32) {
          const int r = c / 16, ch = c % 16, db = ch / 8, cc = ch % 8;
          const uint32_t off = db * (ROWS * 128) + r * 128 + ((cc ^ (r & 7)) * 16);
          cp_async16(dst + off, a.src + static_cast<size_t>(row_of(t, r)) * 128 + ch * 8);
        }
        cp_async_arrive_noinc(full(s));
      } else {
        if (warp == 0 && lane == 0) {
          int r0 = row_of(t, 0);
          if (static_cast<size_t>(r0) + ROWS > a.rows) r0 = 0;
          mbar_arrive_expect_tx(full(s), TILE);
          tma_load_2d(dst, &a.tm_tile, 0, r0, full(s));
          tma_load_2d(dst + ROWS * 128, &a.tm_tile, 64, r0, full(s));
        }
        __syncwarp();
      }
    }
    if (a.mode == MCS_MICRO_CP_ASYNC) asm volatile("cp.async.wait_all;" ::: "memory");
  }
  if (!ok && lane == 0 && !*abort_flag) {
    *abort_flag = 1;
    record_status(a.status, kStatusTimeout);
  }
  __syncthreads();
  // never leave the CTA with a copy still landing in its shared memory
  if (threadIdx.x == 0) {
    volatile int never = 0;
    for (int t = (a.tiles > NS ? a.tiles - NS : 0); t < a.tiles; ++t)
      mbar_wait(full(t % NS), (t / NS) & 1, 2000000000ull, &never);
  }
}

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

bool encode(CUtensorMap *m, const void *base, size_t rows, unsigned box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

unsigned *status_ptr() {
  void *p = nullptr;
  return cudaGetSymbolAddress(&p, g_micro_status) == cudaSuccess ? static_cast<unsigned *>(p) : nullptr;
}

}  // namespace

extern "C" {

mcs_status mcs_micro_gather(const void *src, size_t rows, const int32_t *idx, int ctas, int tiles_per_cta, int mode,
                            int warps, mcs_stream_t stream) {
  if (!src || !idx || rows < ROWS || rows > (1u << 30) || warps < 1 || warps > MAXW || ctas < 1 ||
      tiles_per_cta < 1 || mode < 0 || mode > 2 || (reinterpret_cast<uintptr_t>(src) & 15))
    return MCS_ERR_INVALID_ARG;
  MicroArgs a;
  std::memset(&a, 0, sizeof(a));
  if (!encode(&a.tm_rows, src, rows, 1) || !encode(&a.tm_tile, src, rows, ROWS)) return MCS_ERR_CUDA;
  a.src = static_cast<const bf16 *>(src);
  a.idx = idx;
  a.rows = rows;
  a.tiles = tiles_per_cta;
  a.mode = mode;
  a.warps = warps;
  a.status = status_ptr();
  a.wait_ns = 4000000000ull;
  if (!a.status) return MCS_ERR_CUDA;
  if (cudaFuncSetAttribute(micro_gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess)
    return MCS_ERR_CUDA;
  micro_gather_kernel<<<ctas, THREADS, SMEM, reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? MCS_OK : MCS_ERR_CUDA;
}

mcs_status mcs_micro_last_status(mcs_stream_t stream) {
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

}  // extern "C"
