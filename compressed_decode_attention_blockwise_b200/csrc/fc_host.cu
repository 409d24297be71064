// Host-side pieces of libfc: basis tables, descriptor validation, status
// strings, storage accounting and workspace sizing.
#include <cmath>
#include <mutex>

#include "fc_internal.cuh"

namespace fc {

namespace {

// Orthonormal DCT-II rows (flashcodec-kv README, "Math"):
// M[j][t] = c_j cos(pi / R (t + 1/2) j), c_0 = sqrt(1/R), c_j = sqrt(2/R); the
// same matrix encodes (C = M X) and, transposed, decodes (X = M^T C).
double dct_entry(int R, int j, int t) {
  const double pi = 3.14159265358979323846;
  const double c = (j == 0) ? std::sqrt(1.0 / R) : std::sqrt(2.0 / R);
  return c * std::cos(pi / R * (t + 0.5) * j);
}

// PNG lossless tier (flashcodec-kv README, "Math", PNG bullet): the block is
// stored as its first token (anchor) and the first differences
// Delta_j = x_j - x_{j-1}, so encoding row j takes x_j - x_{j-1} (row 0: x_0)
// and decoding is the cumulative sum x_t = sum_{j <= t} row_j.
double png_encode_entry(int j, int t) {
  if (j == 0) return t == 0 ? 1.0 : 0.0;
  return t == j ? 1.0 : (t == j - 1 ? -1.0 : 0.0);
}
double png_decode_entry(int j, int t) { return j <= t ? 1.0 : 0.0; }

}  // namespace

// Decoding rows: X[t] = sum_j m[j][t] C[j] (fp32; the DCT rows, or the
// cumulative-sum rows of the PNG tier).
void make_basis(int codec, int R, int S, Basis* out) {
  for (int j = 0; j < kMaxS; ++j)
    for (int t = 0; t < kMaxR; ++t) {
      double v = 0.0;
      if (j < S && t < R) v = codec == FC_CODEC_PNG ? png_decode_entry(j, t) : dct_entry(R, j, t);
      out->m[j][t] = static_cast<float>(v);
    }
}

// Encoding rows: C[j] = sum_t m[j][t] X[t] (fp64; the DCT rows, or the
// anchor / first-difference rows of the PNG tier).
void make_basis_f64(int codec, int R, int S, BasisF64* out) {
  for (int j = 0; j < kMaxS; ++j)
    for (int t = 0; t < kMaxR; ++t) {
      double v = 0.0;
      if (j < S && t < R) v = codec == FC_CODEC_PNG ? png_encode_entry(j, t) : dct_entry(R, j, t);
      out->m[j][t] = v;
    }
  out->mirror = codec == FC_CODEC_DCT && R % 2 == 0 ? 1 : 0;
}

int sm_count() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

static bool supported_D(int64_t D) { return D == 32 || D == 64 || D == 128 || D == 256; }

int check_archive(const fc_archive* a) {
  if (!a || !a->coeffs) return FC_ERR_INVALID;
  if (a->coeff_dtype != FC_DTYPE_I8 && a->coeff_dtype != FC_DTYPE_BF16 &&
      a->coeff_dtype != FC_DTYPE_F32)
    return FC_ERR_INVALID;
  const bool quant = a->coeff_dtype == FC_DTYPE_I8;
  if (quant != (a->scales != nullptr)) return FC_ERR_INVALID;
  if (a->B < 1 || a->H < 1 || a->R < 1 || a->S < 1 || a->S > a->R) return FC_ERR_INVALID;
  if (a->codec != FC_CODEC_DCT && a->codec != FC_CODEC_PNG) return FC_ERR_INVALID;
  // the PNG tier keeps every row (S = R) in fp32 (deltas are always fp32)
  if (a->codec == FC_CODEC_PNG && (a->S != a->R || a->R < 2 || a->coeff_dtype != FC_DTYPE_F32))
    return FC_ERR_INVALID;
  if (a->R > kMaxR || a->S > kMaxS || !supported_D(a->D)) return FC_ERR_UNSUPPORTED;
  if (a->capacity < 0 || a->n_blocks < 0 || a->n_blocks > a->capacity) return FC_ERR_INVALID;
  if (!aligned16(a->coeffs) || (quant && !aligned16(a->scales))) return FC_ERR_INVALID;
  const int64_t esz = dtype_size(a->coeff_dtype);
  const int64_t per_head = a->capacity * a->S * a->D;
  if (a->coeff_stride_h < per_head && a->H > 1) return FC_ERR_INVALID;
  if (a->coeff_stride_b < per_head && a->B > 1) return FC_ERR_INVALID;
  if ((a->coeff_stride_b * esz) % 16 || (a->coeff_stride_h * esz) % 16) return FC_ERR_INVALID;
  if (a->coeff_stride_b < 0 || a->coeff_stride_h < 0) return FC_ERR_INVALID;
  if (quant) {
    const int64_t sper = a->capacity * a->S;
    if (a->scale_stride_h < sper && a->H > 1) return FC_ERR_INVALID;
    if (a->scale_stride_b < sper && a->B > 1) return FC_ERR_INVALID;
    if ((a->scale_stride_b * 4) % 16 || (a->scale_stride_h * 4) % 16) return FC_ERR_INVALID;
    if (a->scale_stride_b < 0 || a->scale_stride_h < 0) return FC_ERR_INVALID;
  }
  return FC_OK;
}

int check_tail(const fc_tail* t, const fc_archive* a, bool allow_null_data) {
  if (!t) return FC_ERR_INVALID;
  if (t->dtype != FC_DTYPE_BF16 && t->dtype != FC_DTYPE_F32) return FC_ERR_INVALID;
  if (t->len < 0 || t->len >= a->R) return FC_ERR_INVALID;
  if (!t->data) return allow_null_data && t->len == 0 ? FC_OK : FC_ERR_INVALID;
  if (!aligned16(t->data)) return FC_ERR_INVALID;
  const int64_t esz = dtype_size(t->dtype);
  const int64_t per_head = int64_t(a->R) * a->D;
  if (t->stride_h < per_head && a->H > 1) return FC_ERR_INVALID;
  if (t->stride_b < per_head && a->B > 1) return FC_ERR_INVALID;
  if (t->stride_b < 0 || t->stride_h < 0) return FC_ERR_INVALID;
  if ((t->stride_b * esz) % 16 || (t->stride_h * esz) % 16) return FC_ERR_INVALID;
  return FC_OK;
}

}  // namespace fc

extern "C" {

const char* fc_status_string(int status) {
  switch (status) {
    case FC_OK: return "ok";
    case FC_ERR_INVALID: return "invalid argument (null pointer, shape, stride, alignment or state)";
    case FC_ERR_UNSUPPORTED: return "unsupported size or dtype combination";
    case FC_ERR_CAPACITY: return "archive capacity exhausted; nothing was written";
    case FC_ERR_CUDA: return "CUDA runtime error or kernel launch failure";
    case FC_ERR_DEVICE: return "a kernel reported an error in the workspace status word";
    case FC_ERR_SCRATCH_LIMIT:
      return "request needs more scratch than the library's static array (FC_NOALLOC_SCRATCH_BYTES)";
    default: return "unknown status";
  }
}

int64_t fc_storage_bytes(const fc_archive* arc, const fc_tail* tail) {
  if (fc::check_archive(arc) != FC_OK) return -1;
  const int64_t bh = arc->B * arc->H;
  int64_t total = bh * arc->n_blocks * arc->S * arc->D * fc::dtype_size(arc->coeff_dtype);
  if (arc->coeff_dtype == FC_DTYPE_I8) total += bh * arc->n_blocks * arc->S * 4;
  if (tail) {
    if (fc::check_tail(tail, arc, true) != FC_OK) return -1;
    total += bh * int64_t(tail->len) * arc->D * fc::dtype_size(tail->dtype);
  }
  return total;
}

size_t fc_decode_workspace_bytes(int64_t B, int64_t Hq, int64_t D, int32_t num_splits) {
  if (B < 1 || Hq < 1 || D < 1 || num_splits < 1) return 0;
  return fc::workspace_layout(B, Hq, D, num_splits).total;
}

int fc_workspace_status(void* workspace, size_t workspace_bytes, uint32_t* device_status,
                        fc_stream stream) {
  if (!workspace || workspace_bytes < 256 || !device_status) return FC_ERR_INVALID;
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, workspace, 4, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return FC_ERR_CUDA;
  *device_status = v;
  if (v == 0) return FC_OK;
  e = cudaMemsetAsync(workspace, 0, 4, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return FC_ERR_CUDA;
  return FC_ERR_DEVICE;
}

}  // extern "C"
