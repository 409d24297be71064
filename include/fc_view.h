/*
 * fc_view.h -- structural operations on one libfc stream (archive + raw tail):
 * the reconstructed view, exact removal of trailing tokens, and batch gather
 * (flashcodec-kv 1.0.0, flashcodec/cache.py, _CodecStream.read and
 * _decode_pending, _CodecStream.crop, _CodecStream.select_batch; the HF cache
 * layer's reorder_cache, batch_repeat_interleave and batch_select_indices are
 * batch gathers).
 *
 * Conventions are those of fc.h: caller-owned device memory, element strides,
 * asynchronous on `stream`, host validation before any launch, an fc_status
 * return, no exception and no fallback; host descriptor fields are updated
 * only when a call returns FC_OK.
 */
#ifndef FC_VIEW_H_
#define FC_VIEW_H_

#include "fc.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * fc_read_view -- write the reconstructed (B, H, T, D) view of one stream
 * (flashcodec/cache.py, _CodecStream.read: the archived blocks decompressed
 * and restored to the stream dtype, followed by the raw tail).
 *
 *   arc, tail     the stream; tail may be NULL when the stream has no raw
 *                 tokens (its len is then taken as 0).
 *   first_block   archived blocks [first_block, arc->n_blocks) are decoded:
 *                 row n*R + t of `out` receives
 *                 X_hat = sum_j M[j, t] C_hat[n, j, :] with the DCT-II rows
 *                 M of fc.h and C_hat = code * scale (int8) or the stored
 *                 coefficients, evaluated in fp32 and rounded to out_dtype
 *                 (round to nearest even). 0 <= first_block <= n_blocks.
 *                 Rows below first_block * R are not written, so a caller
 *                 that keeps `out` between calls decodes each archived block
 *                 once (the pages' memoised, append-only view).
 *                 Then the tail's live rows are copied (converted to
 *                 out_dtype) to rows [n_blocks*R, n_blocks*R + len).
 *   out           device, (B, H, out_tokens, D) of out_dtype (FC_DTYPE_BF16
 *                 or FC_DTYPE_F32), 16-byte aligned, element strides
 *                 out_strides[4]: innermost 1, the other three multiples of
 *                 16 bytes; out_tokens >= n_blocks*R + len.
 * One kernel launch (none when nothing is to be written).
 */
int fc_read_view(const fc_archive* arc, const fc_tail* tail,
                 int64_t first_block, void* out, int32_t out_dtype,
                 const int64_t* out_strides, int64_t out_tokens,
                 fc_stream stream);

/*
 * fc_crop -- remove trailing tokens exactly (flashcodec/cache.py,
 * _CodecStream.crop, with the pages' sign convention: a negative count).
 *
 *   tokens_to_remove  <= 0; the last -tokens_to_remove tokens are removed
 *                 (every token when that exceeds the stream's length);
 *                 0 does nothing; a positive value is FC_ERR_INVALID.
 *   arc, tail     the stream (tail required). With
 *                 keep = max(0, n_blocks*R + len - |tokens_to_remove|),
 *                 kb = keep / R and rest = keep mod R: when kb < n_blocks the
 *                 archive keeps its first kb blocks verbatim (n_blocks = kb)
 *                 and the first `rest` tokens of block kb return to tail rows
 *                 [0, rest) as their reconstruction, the values fc_read_view
 *                 writes for them in the tail's dtype; otherwise only the tail
 *                 shrinks. tail->len = rest.
 * One kernel launch when a block returns to the tail, none otherwise.
 */
int fc_crop(fc_archive* arc, fc_tail* tail, int64_t tokens_to_remove,
            fc_stream stream);

/*
 * fc_select_batch -- batch gather (flashcodec/cache.py,
 * _CodecStream.select_batch): batch row i of `dst` becomes batch row idx[i]
 * of `src`, for the archive's live blocks [0, src->n_blocks) (coefficients
 * and scales) and the tail's live rows, byte for byte.
 *
 *   idx           HOST array of n_idx indices, 0 <= idx[i] < src->B;
 *                 repeats are allowed (beam search, repeat-interleave);
 *                 1 <= n_idx <= FC_SELECT_MAX_BATCH.
 *   dst           an archive with B == n_idx and the H, R, S, D and
 *                 coeff_dtype of src, capacity >= src->n_blocks, whose memory
 *                 does not overlap src's; dst->n_blocks becomes
 *                 src->n_blocks.
 *   src_tail, dst_tail   both NULL or both given with the same dtype;
 *                 dst_tail->len becomes src_tail->len.
 * One kernel launch.
 */
#define FC_SELECT_MAX_BATCH 1024
int fc_select_batch(const fc_archive* src, const fc_tail* src_tail,
                    const int64_t* idx, int64_t n_idx, fc_archive* dst,
                    fc_tail* dst_tail, fc_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* FC_VIEW_H_ */
