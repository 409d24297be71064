/*
 * fc.h -- C ABI of libfc: a block-DCT int8 codec for a transformer KV cache and
 * single-token decode attention computed directly on the compressed
 * coefficients, for NVIDIA B200 (sm_100a).
 *
 * Method (flashcodec-kv 1.0.0 README, "Math" and "Materialization-free decode
 * attention"; flashcodec/triton_attention.py; flashcodec/cache.py):
 *   - every complete block of R tokens of a (B, H, T, D) K or V stream is
 *     encoded as C = M X_blk with the orthonormal DCT-II rows
 *     M[j, t] = c_j cos(pi/R (t + 1/2) j), c_0 = sqrt(1/R), c_j = sqrt(2/R),
 *     keeping the S lowest frequencies; the partial last block stays raw;
 *   - int8 storage keeps one fp32 scale per (block, frequency):
 *     scale = max_d |C| / 127, code = clamp(round_half_even(C / scale), -127, 127)
 *     (an all-zero row stores scale 0 and codes 0);
 *   - decode attention never reconstructs K or V: per block s = C_k q,
 *     logits = sigma A s with A = M^T (R x S), an online-softmax update,
 *     w = p A, acc += w C_v; the raw tail joins the same softmax; the pass is
 *     split-K over block chunks and a combine merges the (max, sum, acc)
 *     partials.
 *
 * Conventions for every call:
 *   - All tensors live in device memory owned by the caller. The library never
 *     allocates device memory; scratch comes in through `workspace`.
 *   - Element strides are in ELEMENTS of the tensor's dtype. The innermost
 *     (head_dim) stride is always 1.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and returns an fc_status. Arguments are validated on the
 *     host before anything is launched; on any error nothing is launched and
 *     no descriptor is modified. No exception crosses the ABI.
 *   - Host-side descriptor fields that a call advances (n_blocks, len) are
 *     updated only when the call returns FC_OK.
 *   - There is no fallback path: an unsupported shape or dtype is an error.
 *
 * Supported sizes: D in {32, 64, 128, 256}; 1 <= S <= R <= 32 and S <= 16
 * (the PNG tier: S = R <= 16); Hq a multiple of Hk with G = Hq / Hk in
 * {1, 2, 4, 8, 16}.
 */
#ifndef FC_H_
#define FC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st* fc_stream;

/* Status codes. */
enum {
  FC_OK = 0,
  FC_ERR_INVALID = 1,      /* null pointer, bad shape, stride, alignment or state */
  FC_ERR_UNSUPPORTED = 2,  /* valid but outside the supported sizes/dtypes above */
  FC_ERR_CAPACITY = 3,     /* the archive has too few free blocks; nothing written */
  FC_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  FC_ERR_DEVICE = 5,       /* a kernel reported an error in the workspace status word */
  FC_ERR_SCRATCH_LIMIT = 6 /* fc_decode_attention_noalloc: request exceeds its static scratch */
};

/* fc_decode_attention flags. */
enum {
  FC_DECODE_FUSE_COMBINE = 1, /* the last CTA of each kv head writes `out` */
  FC_DECODE_PORTABLE = 2,     /* force the portable CUDA-core kernel */
  FC_DECODE_OVERLAP = 4,      /* start before the preceding stream work ends */
  FC_DECODE_Q_FINAL = 8,      /* with OVERLAP: q was final before that work began */
  FC_DECODE_TEST_TIMEOUT = 16 /* test hook: make one device wait run out */
};

/* Codecs (fc_archive.codec). */
enum {
  FC_CODEC_DCT = 0, /* block DCT-II, S lowest frequencies (int8 / bf16 / fp32) */
  FC_CODEC_PNG = 1  /* lossless PNG tier: anchor + fp32 first differences */
};

/* Element types. */
enum {
  FC_DTYPE_F32 = 0,
  FC_DTYPE_BF16 = 1,
  FC_DTYPE_I8 = 2
};

/*
 * Compressed archive of one K or V stream (flashcodec/cache.py, _CodecStream:
 * coefficients (B, H, capacity, K, D), int8 codes with fp32 scales
 * (B, H, capacity, K, 1) when quantised, else the stream dtype).
 *
 *   coeffs  device, (B, H, capacity, S, D) of coeff_dtype. Within one (b, h)
 *           the (capacity, S, D) block is contiguous: block stride S*D,
 *           frequency stride D, element stride 1. 16-byte aligned.
 *   scales  device, (B, H, capacity, S) fp32, contiguous per (b, h); required
 *           when coeff_dtype == FC_DTYPE_I8, must be NULL otherwise.
 *   coeff_dtype  FC_DTYPE_I8 (quantised), FC_DTYPE_BF16 or FC_DTYPE_F32.
 *   codec        FC_CODEC_DCT: rows C = M X_blk with the DCT-II rows M.
 *                FC_CODEC_PNG (flashcodec-kv README, "Math", PNG bullet; the
 *                lossless tier, keep_ratio 1.0): S == R rows per block in
 *                fp32, row 0 the block's first token (the anchor, converted
 *                exactly) and row j >= 1 the first difference
 *                x_j - x_{j-1} rounded once to fp32; decoding is the
 *                cumulative sum x_t = sum_{j <= t} row_j, and decode attention
 *                takes the same per-block steps with A[t][j] = 1 for j <= t.
 *                Every call of this header and of fc_view.h serves both
 *                codecs; the tensor-core kernel serves the DCT only.
 *   n_blocks     archived blocks per (b, h), 0 <= n_blocks <= capacity; the
 *                library advances it when it archives blocks.
 *   *_stride_b / *_stride_h  element strides of the batch and head axes;
 *                coefficient strides times the element size must be multiples
 *                of 16 bytes.
 * Archived blocks are never rewritten by any call (causal safety).
 */
typedef struct fc_archive {
  void* coeffs;
  float* scales;
  int32_t coeff_dtype;
  int32_t R;
  int32_t S;
  int32_t codec;
  int64_t B, H, D;
  int64_t capacity;
  int64_t n_blocks;
  int64_t coeff_stride_b, coeff_stride_h;
  int64_t scale_stride_b, scale_stride_h;
} fc_archive;

/*
 * Raw tail of one stream: the tokens of the incomplete last block, kept at the
 * input precision (flashcodec/cache.py, _CodecStream.raw).
 *
 *   data    device, (B, H, R, D) of dtype; rows [0, len) are live. Token
 *           stride D, element stride 1. 16-byte aligned.
 *   dtype   FC_DTYPE_BF16 or FC_DTYPE_F32 (the stream's input dtype).
 *   len     0 <= len < R; advanced by fc_append_step / fc_compress_blocks.
 */
typedef struct fc_tail {
  void* data;
  int32_t dtype;
  int32_t len;
  int64_t stride_b, stride_h;
} fc_tail;

/*
 * fc_compress_blocks -- archive the complete blocks of a prefill
 * (flashcodec/cache.py, _CodecStream.append and _archive: the full-block head
 * is compressed and written as one slice; the remainder stays raw).
 *
 *   x        device, (B, H, T, D) tokens of x_dtype (FC_DTYPE_BF16 or
 *            FC_DTYPE_F32) with element strides x_strides[4]
 *            (x_strides[3] == 1). Read only.
 *   T        tokens in x, T >= 0.
 *   arc      archive; the floor(T / R) complete blocks go to slots
 *            [arc->n_blocks, arc->n_blocks + floor(T / R)), then n_blocks
 *            advances. Needs capacity for all of them, else FC_ERR_CAPACITY.
 *   tail     optional (may be NULL). When given it must have len == 0 and the
 *            same dtype as x; the T mod R remaining tokens are copied into its
 *            rows [0, T mod R) and len is set to T mod R. When NULL the caller
 *            keeps the remainder itself.
 * One kernel launch (none when there is nothing to do).
 */
int fc_compress_blocks(const void* x, int32_t x_dtype, const int64_t* x_strides,
                       int64_t T, fc_archive* arc, fc_tail* tail,
                       fc_stream stream);

/*
 * fc_append_step -- append one decode token to the K and V streams
 * (flashcodec/cache.py, CodecKVCache.decode_step / _CodecStream.append with a
 * single token): the token is written to tail row `len`; when that fills the
 * block (len + 1 == R) the R tail tokens are compressed into archive slot
 * n_blocks, n_blocks advances and len returns to 0.
 *
 *   k_new, v_new   device, (B, H, 1, D) of `dtype` (the tails' dtype), element
 *                  strides k_strides[4] / v_strides[4], innermost 1.
 *   ka, va         K and V archives (same B, H, R, S, D, n_blocks).
 *   kt, vt         K and V tails (same len).
 * FC_ERR_CAPACITY (nothing written) when a block would complete with
 * n_blocks == capacity: grow the archive (fc_archive_copy_prefix) and retry.
 * One kernel launch for both streams.
 */
int fc_append_step(const void* k_new, const void* v_new, int32_t dtype,
                   const int64_t* k_strides, const int64_t* v_strides,
                   fc_archive* ka, fc_archive* va, fc_tail* kt, fc_tail* vt,
                   fc_stream stream);

/*
 * fc_archive_copy_prefix -- copy the live blocks [0, src->n_blocks) of every
 * (b, h) from src into dst and set dst->n_blocks = src->n_blocks: the copy
 * step of the archive's geometric growth (flashcodec/cache.py,
 * _CodecStream._grow: capacity starts at 16 blocks and doubles; the old data
 * is copied verbatim). src and dst must agree on B, H, R, S, D and dtype, and
 * dst->capacity >= src->n_blocks. One kernel launch.
 */
int fc_archive_copy_prefix(const fc_archive* src, fc_archive* dst,
                           fc_stream stream);

/*
 * fc_decode_plan -- the split count fc_decode_attention uses when called with
 * num_splits == 0 for these archives on the current device (chosen to fill the
 * GPU's SMs; results do not depend on it beyond rounding).
 */
int fc_decode_plan(const fc_archive* ka, const fc_tail* kt, int64_t Hq,
                   int32_t* num_splits_out);

/*
 * fc_decode_kernel -- which kernel fc_decode_attention / fc_decode_step use
 * for these archives, Hq and flags on the current device: FC_KERNEL_TENSOR_CORE
 * (5th-generation tensor cores, the int8 paths of the header's supported
 * sizes) or FC_KERNEL_CUDA_CORE (the portable kernel). Host query only; the
 * results of the two kernels agree to rounding.
 */
enum { FC_KERNEL_CUDA_CORE = 0, FC_KERNEL_TENSOR_CORE = 1 };
int fc_decode_kernel(const fc_archive* ka, const fc_archive* va, int64_t Hq,
                     int32_t flags, int32_t* kind_out);

/*
 * fc_decode_workspace_bytes -- bytes of workspace fc_decode_attention and
 * fc_combine need for (B, Hq, D, num_splits): a status word, one ticket per
 * (b, kv head), and the fp32 partials (max, sum, acc[D]) per (b, q head,
 * split). Returns 0 for invalid sizes.
 */
size_t fc_decode_workspace_bytes(int64_t B, int64_t Hq, int64_t D,
                                 int32_t num_splits);

/*
 * fc_decode_attention -- single-token decode attention on the compressed
 * archive plus the raw tail (flashcodec/triton_attention.py, split and combine
 * kernels; README "Materialization-free decode attention").
 *
 *   q          device, (B, Hq, 1, D) of q_dtype (FC_DTYPE_BF16 or FC_DTYPE_F32),
 *              element strides q_strides[4], innermost 1. Query head hq reads
 *              kv head hq / G, G = Hq / Hk.
 *   ka, va     K and V archives; kt, vt their tails (may be NULL when empty).
 *              Every archived block and every live tail token is attended;
 *              there is no mask. n_blocks == 0 is allowed (tail-only softmax);
 *              n_blocks == 0 with an empty tail is FC_ERR_INVALID.
 *   softmax_scale   sigma; <= 0 selects D^-0.5.
 *   num_splits      split-K chunks per kv head, 0 = fc_decode_plan's
 *                   choice. Chunks partition each kv head's blocks
 *                   contiguously and in order: c * chunk .. (c + 1) * chunk
 *                   with chunk = ceil(n / num_splits) of the kernel's units
 *                   (blocks; whole 128-row coefficient tiles on the
 *                   tensor-core kernel), so the last chunk may be shorter or
 *                   empty; the raw tail belongs to the last chunk.
 *   flags      FC_DECODE_FUSE_COMBINE: the last CTA to finish a kv head
 *              merges the partials and writes `out` (one launch, no
 *              spin-waits: an atomic ticket); without it only the partials
 *              are written and fc_combine produces `out`.
 *              FC_DECODE_PORTABLE: use the portable CUDA-core kernel even
 *              where the tensor-core kernel applies (DCT codec, int8 K and
 *              V, D = 128, (S, R / S) in {(1, 4), (1, 8), (2, 4), (2, 8),
 *              (4, 2), (4, 4), (8, 2)}, G in {1, 2, 4, 8} with
 *              max(1, G / S) R <= 32, at least one archived block;
 *              fc_decode_kernel reports the choice).
 *              FC_DECODE_OVERLAP (tensor-core kernel; ignored otherwise):
 *              launch as a programmatic dependent of the preceding work on
 *              `stream`. The kernel then streams archive blocks
 *              [0, n_blocks - 1) while that work is still running, and waits
 *              for it before it reads q, the tails or block n_blocks - 1 and
 *              before it writes the workspace or `out`. Precondition: no
 *              work still in flight on the stream writes archive blocks
 *              below n_blocks - 1. A decode loop of fc_append_step and
 *              fc_decode_attention meets it (an append writes at most block
 *              n_blocks - 1 and the tails); a fc_compress_blocks of the same
 *              archive queued just before does not. Pure scheduling: the
 *              results are those of a launch without the flag.
 *              FC_DECODE_Q_FINAL (with FC_DECODE_OVERLAP): q already held its
 *              final values when the preceding kernel on the stream began
 *              executing (it was written by work that completed before that
 *              kernel started, e.g. a projection followed by a plain
 *              fc_append_step launch). The kernel then also reads q and
 *              computes over blocks [0, n_blocks - 1) before the preceding
 *              work completes; it still waits before block n_blocks - 1,
 *              the tails, the workspace and `out`. Ignored without
 *              FC_DECODE_OVERLAP.
 *              FC_DECODE_TEST_TIMEOUT (fc_decode_attention only; a test
 *              hook for the error path): every CTA of the tensor-core
 *              kernel makes one wait on a barrier phase that nothing
 *              completes, with a limit of about 2^20 clock cycles instead
 *              of the usual ~2 s. The wait runs out, the CTA records the
 *              error in the workspace status word, stops issuing loads and
 *              MMAs, drains the ones in flight, frees its TMEM and returns;
 *              the tickets still return to zero, so the workspace serves
 *              the next call. The call returns FC_OK (the launch worked);
 *              fc_workspace_status then reports FC_ERR_DEVICE and `out` is
 *              unspecified. FC_ERR_UNSUPPORTED where the tensor-core kernel
 *              does not apply (or with FC_DECODE_PORTABLE); FC_ERR_INVALID
 *              with FC_DECODE_FUSE_COMBINE and a single split (no
 *              workspace, so no status word).
 *   workspace       device, >= fc_decode_workspace_bytes(B, Hq, D, splits)
 *                   bytes, 256-byte aligned. Its first 256 + 4*B*Hq bytes
 *                   (status word and tickets) must be zero before the first
 *                   call; every completed call leaves them zero again. Calls
 *                   that share a workspace must not overlap on the GPU.
 *   out        device, (B, Hq, 1, D) of out_dtype (FC_DTYPE_F32 or
 *              FC_DTYPE_BF16), element strides out_strides[4], innermost 1.
 * One kernel launch.
 */
int fc_decode_attention(const void* q, int32_t q_dtype, const int64_t* q_strides,
                        int64_t Hq, const fc_archive* ka, const fc_archive* va,
                        const fc_tail* kt, const fc_tail* vt,
                        float softmax_scale, int32_t num_splits,
                        int32_t flags, void* workspace,
                        size_t workspace_bytes, void* out, int32_t out_dtype,
                        const int64_t* out_strides, fc_stream stream);

/*
 * fc_decode_step -- one decode step: fc_append_step(k_new, v_new, ...)
 * followed by fc_decode_attention(q, ...) over the updated streams, with the
 * same results (the archive bitwise; `out` up to the rounding of the new
 * token's or block's softmax terms) in one kernel launch where the
 * tensor-core kernel applies (flashcodec/cache.py, _CodecStream.append, then
 * flashcodec/triton_attention.py, the split kernel: the pages run these as
 * separate calls; fusing them is this library's). In the fused launch the
 * last chunk's CTA of each (b, kv head) folds the new token into the softmax
 * as a raw token and stores it at tail row len, or, when the token completes
 * a block, encodes that block (tail rows 0..R-2 and the token) into archive
 * slot n_blocks with the codec's own device code and folds it in the
 * coefficient domain. Elsewhere (portable flag, no archived block yet, other
 * dtypes) it issues the two calls.
 *   k_new, v_new, new_dtype, k_strides, v_strides: as in fc_append_step;
 *              new_dtype must equal the tails' dtype.
 *   ka, va, kt, vt: as in fc_append_step (tails required); on success the
 *              host descriptors are updated as fc_append_step does.
 *   other arguments: as in fc_decode_attention; FC_DECODE_OVERLAP also
 *              covers k_new and v_new (read after the dependency wait).
 * Errors as fc_append_step (FC_ERR_CAPACITY leaves everything unchanged) and
 * fc_decode_attention.
 */
int fc_decode_step(const void* q, int32_t q_dtype, const int64_t* q_strides, int64_t Hq,
                   const void* k_new, const void* v_new, int32_t new_dtype,
                   const int64_t* k_strides, const int64_t* v_strides, fc_archive* ka,
                   fc_archive* va, fc_tail* kt, fc_tail* vt, float softmax_scale,
                   int32_t num_splits, int32_t flags, void* workspace,
                   size_t workspace_bytes, void* out, int32_t out_dtype,
                   const int64_t* out_strides, fc_stream stream);

/*
 * fc_decode_step_host -- fc_decode_step fed from and returning to HOST
 * memory, for a serving loop whose tokens and queries arrive on the host.
 * When both host buffers are pinned memory the device can address (every
 * pinned allocation under unified addressing), the kernels read the inputs
 * and write the output there directly; otherwise one host-to-device copy of
 * the inputs into `staging`, the fused step and one device-to-host copy of
 * the output are queued. All work is on `stream`; the output is complete
 * once `stream` has reached it.
 *   in_host    host, the contiguous block [k_new | v_new | q]: k_new and
 *              v_new (B, H, 1, D), q (B, Hq, 1, D), each contiguous, of
 *              io_dtype (FC_DTYPE_BF16 or FC_DTYPE_F32, the tails' dtype).
 *   out_host   host, (B, Hq, 1, D) contiguous of out_dtype.
 *   staging    device, >= fc_decode_step_staging_bytes(...), 256-byte
 *              aligned: the inputs' and the output's device copies.
 *   other arguments as in fc_decode_step (the archives and tails are
 *              updated in the same way).
 */
size_t fc_decode_step_staging_bytes(int64_t B, int64_t H, int64_t Hq, int64_t D,
                                    int32_t io_dtype, int32_t out_dtype);
int fc_decode_step_host(const void* in_host, void* out_host, void* staging,
                        size_t staging_bytes, int32_t io_dtype, int32_t out_dtype,
                        int64_t Hq, fc_archive* ka, fc_archive* va, fc_tail* kt,
                        fc_tail* vt, float softmax_scale, int32_t num_splits,
                        int32_t flags, void* workspace, size_t workspace_bytes,
                        fc_stream stream);

/*
 * fc_decode_step_layers -- the fused decode steps of n_layers independent
 * streams in ONE kernel launch: layer i does fc_decode_step(layers[i].q,
 * layers[i].k_new, layers[i].v_new, ...) with the results of that call
 * (bitwise: every CTA runs the single call's code on its layer). The launch's
 * CTAs are every layer's (kv head, chunk) pieces; the hardware starts the
 * next layer's pieces as SMs free up, so one launch's start-up and one
 * drain are paid instead of n_layers (flashcodec-kv README,
 * "Materialization-free decode attention": the split/combine launches are
 * the remaining end-to-end gap). Every query and new token must be final
 * when the launch starts (the layers of a step whose queries are known, or
 * the sequences of a serving batch with their own caches); a model whose
 * layer l + 1 query depends on layer l's output calls fc_decode_step per
 * layer.
 *   n_layers   1 .. FC_MAX_LAYERS.
 *   layers     per layer: q (B, Hq, 1, D) and its strides; k_new / v_new
 *              (B, H, 1, D) and strides; the K and V archives and tails
 *              (updated on success as fc_decode_step does); a workspace of
 *              fc_decode_workspace_bytes for its split; out (B, Hq, 1, D) and
 *              strides. No two layers share an archive, tail or workspace.
 *   q_dtype, new_dtype, out_dtype, Hq, softmax_scale, num_splits: as in
 *              fc_decode_step, shared by all layers.
 *   flags      FC_DECODE_FUSE_COMBINE, FC_DECODE_OVERLAP and
 *              FC_DECODE_Q_FINAL as in fc_decode_attention, for every layer
 *              (with the overlap flags the launch is a programmatic dependent
 *              of the preceding stream work, e.g. the previous step's
 *              launch, under the same precondition); FC_DECODE_PORTABLE is
 *              FC_ERR_INVALID.
 * Every layer must be a tensor-core fused step (int8 K and V, D = 128, the
 * sizes fc_decode_attention lists for that kernel) with the same G, S and
 * R, else FC_ERR_UNSUPPORTED; FC_ERR_CAPACITY for any layer leaves every
 * layer unchanged. One kernel launch.
 */
#define FC_MAX_LAYERS 16
typedef struct fc_layer_step {
  const void* q;
  int64_t q_strides[4];
  const void* k_new;
  const void* v_new;
  int64_t k_strides[4];
  int64_t v_strides[4];
  fc_archive* ka;
  fc_archive* va;
  fc_tail* kt;
  fc_tail* vt;
  void* workspace;
  size_t workspace_bytes;
  void* out;
  int64_t out_strides[4];
} fc_layer_step;
int fc_decode_step_layers(int32_t n_layers, fc_layer_step* layers, int32_t q_dtype,
                          int32_t new_dtype, int32_t out_dtype, int64_t Hq,
                          float softmax_scale, int32_t num_splits, int32_t flags,
                          fc_stream stream);

/*
 * fc_combine -- merge split-K partials left in `workspace` by
 * fc_decode_attention without FC_DECODE_FUSE_COMBINE (flashcodec/triton_attention.py,
 * combine kernel): M = max_c m_c, L = sum_c l_c e^(m_c - M),
 * out = sum_c acc_c e^(m_c - M) / L; chunks with l_c = 0 are skipped.
 * Sizes must match the producing call. One kernel launch.
 */
int fc_combine(const void* workspace, size_t workspace_bytes, int64_t B,
               int64_t Hq, int64_t D, int32_t num_splits, void* out,
               int32_t out_dtype, const int64_t* out_strides, fc_stream stream);

/*
 * fc_decode_attention_noalloc -- fc_decode_attention (fused combine) for
 * callers that cannot hand the library a workspace: a C host that runs inside
 * a fixed device-memory budget with no allocator of its own, or a serving
 * loop that must not call cudaMalloc per step because the call synchronises
 * the device. The paper has no counterpart; this is an interface convenience.
 *
 * Instead of a caller workspace the call uses one file-scope device array of
 * FC_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until the
 * process exits. It calls no cudaMalloc, cudaFree or allocating routine. The
 * first call on a device resolves the array's device address with
 * cudaGetSymbolAddress (once per device, with that device current); make that
 * first call before any stream capture. Every call shares the array and
 * clears its tickets on `stream` before the kernel, so calls whose executions
 * overlap on the GPU (other streams, other host threads) race; serialise
 * them. The array's status word is not cleared by these calls: a kernel error
 * (a bounded wait that gave up) stays recorded until fc_noalloc_status reads
 * and clears it. Arguments and results as in fc_decode_attention; returns
 * FC_ERR_SCRATCH_LIMIT, launching nothing, when
 * fc_decode_workspace_bytes(B, Hq, D, splits) exceeds the array.
 */
#define FC_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
int fc_decode_attention_noalloc(const void* q, int32_t q_dtype, const int64_t* q_strides,
                                int64_t Hq, const fc_archive* ka, const fc_archive* va,
                                const fc_tail* kt, const fc_tail* vt, float softmax_scale,
                                int32_t num_splits, void* out, int32_t out_dtype,
                                const int64_t* out_strides, fc_stream stream);

/*
 * fc_noalloc_status -- fc_workspace_status for the static scratch array of
 * fc_decode_attention_noalloc on the current device: synchronises `stream`,
 * stores the status word in *device_status (0 = no fc_decode_attention_noalloc
 * kernel on this device reported a problem since the last read) and clears
 * it. Returns FC_ERR_DEVICE when it was nonzero. Allocates nothing.
 */
int fc_noalloc_status(uint32_t* device_status, fc_stream stream);

/*
 * fc_workspace_status -- synchronise `stream`, read the workspace status word
 * into *device_status (0 = no kernel reported a problem) and clear it.
 * Returns FC_ERR_DEVICE when it was nonzero.
 */
int fc_workspace_status(void* workspace, size_t workspace_bytes,
                        uint32_t* device_status, fc_stream stream);

/*
 * fc_storage_bytes -- logical storage of one stream: the live archive region
 * (n_blocks blocks of coefficients, plus their fp32 scales when quantised) and
 * the live raw tail, excluding idle capacity (flashcodec/cache.py,
 * _CodecStream.storage_bytes). Host arithmetic only; tail may be NULL.
 * Returns -1 for an invalid descriptor.
 */
int64_t fc_storage_bytes(const fc_archive* arc, const fc_tail* tail);

/* fc_status_string -- static description of a status code. */
const char* fc_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FC_H_ */
