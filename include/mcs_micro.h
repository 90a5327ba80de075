/*
 * mcs_micro.h -- measurement-only entry points of libmcs_micro.so.
 *
 * The reused step of MC-Sparse brings index-listed K and V rows into shared
 * memory before each tensor-core tile (cnshai.top "output-aware sparse
 * attention / KV cache" post, "What Trips People Up": gathering irregular
 * rows is what token-level selection costs).  The rate at which one SM can do
 * that bounds the step whenever the tensor cores are not the limit, so it is
 * measured on its own here.  The pages describe no such call; it exists so
 * the ceiling the step is reported against can be re-measured on any box.
 * The exponential and MMA rates are measured the same way: the softmax's
 * MUFU work and the tensor pipe's MMA rate are the other two ceilings of the
 * step.  Nothing here is on the hot path.
 */
#ifndef MCS_MICRO_H_
#define MCS_MICRO_H_

#include "mcs.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MCS_MICRO_GATHER4 = 0,   /* TMA tile::gather4, four 128-byte row pieces per operation */
  MCS_MICRO_CP_ASYNC = 1,  /* cp.async, 16 bytes per thread per operation               */
  MCS_MICRO_TILE = 2       /* TMA tile loads of 128 contiguous rows (no index list)      */
} mcs_micro_mode;

/*
 * mcs_micro_gather -- each CTA (one per SM, `ctas` of them) streams
 * `tiles_per_cta` tiles of 128 rows x 256 bytes (bf16 rows of d = 128) from
 * `src` into a four-slot shared-memory ring, issued by `warps` producer warps
 * (1..8) in the given mode; one consumer thread frees each slot as soon as it
 * is full.  Rows of tile t of CTA c are idx[(c * tiles_per_cta + t) * 128 +
 * r]; for MCS_MICRO_TILE only the first index of each tile is used and the
 * tile is rows [idx, idx + 128).
 * src: bf16 [rows, 128] device memory, 16-byte aligned.  idx: int32 device
 * memory of ctas * tiles_per_cta * 128 entries in [0, rows) (an entry out of
 * range is replaced by row 0 and recorded as MCS_ERR_BAD_META in the device
 * status word that mcs_last_device_status of libmcs.so does NOT see: read it
 * with mcs_micro_last_status).  Bytes moved: ctas * tiles_per_cta * 32768.
 * Asynchronous on `stream`; INVALID_ARG for null pointers, rows < 128,
 * warps outside 1..8, ctas < 1 or tiles_per_cta < 1.
 */
mcs_status mcs_micro_gather(const void *src, size_t rows, const int32_t *idx, int ctas, int tiles_per_cta,
                            int mode, int warps, mcs_stream_t stream);

/*
 * mcs_micro_ex2 -- the MUFU exponential rate: `ctas` CTAs of `warps` warps
 * (1..32) each run 8 independent chains of `iters` steps v = 2^v - 1.5
 * (ex2.approx, the instruction every softmax here uses) per thread.
 * cycles: device array of 2 * ctas entries; entry c receives CTA c's SM
 * cycles (clock64) for its whole loop; the second half is scratch.
 * Exponentials per CTA: warps * 32 * iters * 8.  Asynchronous; INVALID_ARG
 * for a null pointer or out-of-range counts.
 */
mcs_status mcs_micro_ex2(int ctas, int warps, int iters, unsigned long long *cycles, mcs_stream_t stream);

/*
 * mcs_micro_mma -- the tcgen05 MMA rate of one SM: in each of `ctas` CTAs one
 * warp issues `batches` x 8 x `chains` back-to-back MMAs of kind::f16 (bf16
 * in, fp32 accumulate), from one elected lane per MMA as the reused step
 * does, and times them (clock64) to the completion of the last one.  The
 * MMAs accumulate into `chains` TMEM accumulators, each k16 step issued to
 * every accumulator in turn (1 chain: every MMA depends on the one before;
 * more: independent chains interleaved; at most 4 for shape 0, 2 otherwise).  shape 0: SS, M = 128, N = 64 (the step's Q.K^T); 1: TS, M = 128,
 * N = 128 with A read from TMEM and B MN-major (the step's P.V); 2: SS,
 * M = 128, N = 128.  load 0: nothing else runs; 1: eight other warps of the
 * CTA issue MUFU exponentials meanwhile; 2: they issue FMAs (the pipes the
 * softmax occupies while the MMAs run).  out: device array of 3 * ctas + 1
 * entries: per CTA (cycles, MMAs issued, 1 if the completion wait ran out);
 * the last entry is scratch.  Operands are zeros.  Asynchronous;
 * INVALID_ARG for a null pointer or out-of-range arguments.
 */
mcs_status mcs_micro_mma(int ctas, int shape, int batches, int load, int chains, unsigned long long *out,
                         mcs_stream_t stream);

/* Synchronise `stream`, then read and clear the micro library's status word. */
mcs_status mcs_micro_last_status(mcs_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MCS_MICRO_H_ */
