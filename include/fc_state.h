/*
 * fc_state.h -- exact save and restore of one libfc stream (archive + raw
 * tail) through host memory.
 *
 * The pages' cache hands its state out as reconstructed views and rebuilds a
 * cache by sending them through the codec again (flashcodec/cache.py,
 * FlashCodecCache.to_legacy_cache / from_legacy_cache), which is lossy a
 * second time. These calls move the stored bytes instead, so that a restored
 * stream is bitwise the saved one: the live coefficients (codes or stored
 * coefficients), their fp32 scales and the live raw tail rows, behind a small
 * header that records the stream's geometry.
 *
 * Image layout (host memory, native byte order):
 *   fc_state_header (below)
 *   coefficients   (B, H, n_blocks, S, D) of coeff_dtype, contiguous
 *   scales         (B, H, n_blocks, S) fp32, contiguous (int8 archives only)
 *   tail rows      (B, H, tail_len, D) of tail_dtype, contiguous
 *
 * Conventions are those of fc.h: caller-owned memory, asynchronous on
 * `stream`, host validation before any copy, an fc_status return, no
 * exception; descriptor fields are updated only when a call returns FC_OK.
 */
#ifndef FC_STATE_H_
#define FC_STATE_H_

#include "fc.h"

#ifdef __cplusplus
extern "C" {
#endif

#define FC_STATE_MAGIC "FCSTATE1"

typedef struct fc_state_header {
  char magic[8];        /* FC_STATE_MAGIC without its terminating zero */
  int32_t version;      /* 1 */
  int32_t coeff_dtype;  /* as fc_archive */
  int32_t tail_dtype;   /* as fc_tail */
  int32_t R, S;
  int32_t tail_len;
  int64_t B, H, D;
  int64_t n_blocks;
  int64_t coeff_bytes, scale_bytes, tail_bytes;  /* payload sizes */
} fc_state_header;

/*
 * fc_state_bytes -- size of the image of (arc, tail): header plus payload.
 * tail may be NULL (no raw tokens). Returns 0 for an invalid descriptor.
 */
size_t fc_state_bytes(const fc_archive* arc, const fc_tail* tail);

/*
 * fc_state_save -- write the image of the stream into host memory `dst`
 * (dst_bytes >= fc_state_bytes). The header is written before the call
 * returns; the payload is copied from the device by cudaMemcpy2DAsync calls
 * on `stream` (one per batch row and part; pinned `dst` makes them
 * asynchronous), so `dst` is complete once `stream` has reached them. The
 * stream itself is not modified.
 */
int fc_state_save(const fc_archive* arc, const fc_tail* tail, void* dst,
                  size_t dst_bytes, fc_stream stream);

/*
 * fc_state_restore -- load an image from host memory `src` into the stream
 * (arc, tail): the header must match the stream's B, H, R, S, D, coefficient
 * dtype and (when the image holds raw tokens) tail dtype, the archive needs
 * capacity >= the image's n_blocks, else FC_ERR_INVALID / FC_ERR_CAPACITY
 * with nothing copied. On FC_OK the copies are queued on `stream` and
 * arc->n_blocks and tail->len are set from the image; archive slots past
 * n_blocks and tail rows past len are not touched. tail may be NULL only
 * when the image holds no raw tokens.
 */
int fc_state_restore(const void* src, size_t src_bytes, fc_archive* arc,
                     fc_tail* tail, fc_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* FC_STATE_H_ */
