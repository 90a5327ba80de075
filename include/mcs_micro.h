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
 * Nothing here is on the hot path.
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

/* Synchronise `stream`, then read and clear the micro library's status word. */
mcs_status mcs_micro_last_status(mcs_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MCS_MICRO_H_ */
