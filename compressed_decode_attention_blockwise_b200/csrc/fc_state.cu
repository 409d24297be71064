// Exact save and restore of one stream through host memory (fc_state.h):
// plain strided copies of the live archive and raw tail, no kernel.
#include <cstring>

#include "fc_internal.cuh"
#include "fc_state.h"

namespace fc {
namespace {

struct Parts {
  int64_t coeff_row;   // bytes of one (b, h) run of live coefficients
  int64_t scale_row;   // ... of live scales
  int64_t tail_row;    // ... of live tail rows
  int64_t coeff, scale, tail;  // totals
};

Parts parts_of(const fc_archive* a, int64_t n_blocks, int tail_len, int tail_dtype) {
  Parts p;
  const int64_t bh = a->B * a->H;
  p.coeff_row = n_blocks * a->S * a->D * dtype_size(a->coeff_dtype);
  p.scale_row = a->coeff_dtype == FC_DTYPE_I8 ? n_blocks * a->S * 4 : 0;
  p.tail_row = int64_t(tail_len) * a->D * (tail_len ? dtype_size(tail_dtype) : 0);
  p.coeff = bh * p.coeff_row;
  p.scale = bh * p.scale_row;
  p.tail = bh * p.tail_row;
  return p;
}

// one strided copy per batch row: H runs of `width` bytes, `dpitch` /
// `spitch` apart (in elements of `esz` bytes for the device side)
int copy_runs(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width, size_t height,
              cudaMemcpyKind kind, cudaStream_t stream) {
  if (width == 0 || height == 0) return FC_OK;
  return cuda_status(cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, height, kind, stream));
}

// device pitch of the head axis in bytes (any value >= width when H == 1)
size_t head_pitch(int64_t stride_h, int64_t H, size_t width, int esz) {
  return H > 1 ? size_t(stride_h) * size_t(esz) : width;
}

}  // namespace
}  // namespace fc

using namespace fc;

extern "C" size_t fc_state_bytes(const fc_archive* arc, const fc_tail* tail) {
  if (check_archive(arc) != FC_OK) return 0;
  if (tail && check_tail(tail, arc, true) != FC_OK) return 0;
  const int len = tail ? tail->len : 0;
  const Parts p = parts_of(arc, arc->n_blocks, len, tail ? tail->dtype : FC_DTYPE_BF16);
  return sizeof(fc_state_header) + size_t(p.coeff + p.scale + p.tail);
}

extern "C" int fc_state_save(const fc_archive* arc, const fc_tail* tail, void* dst, size_t dst_bytes,
                             fc_stream stream) {
  int st = check_archive(arc);
  if (st != FC_OK) return st;
  if (tail) {
    st = check_tail(tail, arc, true);
    if (st != FC_OK) return st;
  }
  if (!dst) return FC_ERR_INVALID;
  const int len = tail ? tail->len : 0;
  const int tdt = tail ? tail->dtype : FC_DTYPE_BF16;
  const Parts p = parts_of(arc, arc->n_blocks, len, tdt);
  if (dst_bytes < sizeof(fc_state_header) + size_t(p.coeff + p.scale + p.tail)) return FC_ERR_INVALID;
  fc_state_header hd;
  std::memset(&hd, 0, sizeof(hd));
  std::memcpy(hd.magic, FC_STATE_MAGIC, 8);
  hd.version = 1;
  hd.coeff_dtype = arc->coeff_dtype;
  hd.tail_dtype = tdt;
  hd.R = arc->R;
  hd.S = arc->S;
  hd.tail_len = len;
  hd.B = arc->B;
  hd.H = arc->H;
  hd.D = arc->D;
  hd.n_blocks = arc->n_blocks;
  hd.coeff_bytes = p.coeff;
  hd.scale_bytes = p.scale;
  hd.tail_bytes = p.tail;
  std::memcpy(dst, &hd, sizeof(hd));
  uint8_t* out = static_cast<uint8_t*>(dst) + sizeof(hd);
  const int cesz = dtype_size(arc->coeff_dtype);
  for (int64_t b = 0; b < arc->B; ++b) {
    const uint8_t* cs = static_cast<const uint8_t*>(arc->coeffs) + b * arc->coeff_stride_b * cesz;
    st = copy_runs(out + b * arc->H * p.coeff_row, size_t(p.coeff_row), cs,
                   head_pitch(arc->coeff_stride_h, arc->H, size_t(p.coeff_row), cesz), size_t(p.coeff_row),
                   size_t(arc->H), cudaMemcpyDeviceToHost, stream);
    if (st != FC_OK) return st;
    if (p.scale_row) {
      const uint8_t* ss = reinterpret_cast<const uint8_t*>(arc->scales) + b * arc->scale_stride_b * 4;
      st = copy_runs(out + p.coeff + b * arc->H * p.scale_row, size_t(p.scale_row), ss,
                     head_pitch(arc->scale_stride_h, arc->H, size_t(p.scale_row), 4), size_t(p.scale_row),
                     size_t(arc->H), cudaMemcpyDeviceToHost, stream);
      if (st != FC_OK) return st;
    }
    if (p.tail_row) {
      const int tesz = dtype_size(tdt);
      const uint8_t* ts = static_cast<const uint8_t*>(tail->data) + b * tail->stride_b * tesz;
      st = copy_runs(out + p.coeff + p.scale + b * arc->H * p.tail_row, size_t(p.tail_row), ts,
                     head_pitch(tail->stride_h, arc->H, size_t(p.tail_row), tesz), size_t(p.tail_row),
                     size_t(arc->H), cudaMemcpyDeviceToHost, stream);
      if (st != FC_OK) return st;
    }
  }
  return FC_OK;
}

extern "C" int fc_state_restore(const void* src, size_t src_bytes, fc_archive* arc, fc_tail* tail,
                                fc_stream stream) {
  int st = check_archive(arc);
  if (st != FC_OK) return st;
  if (!src || src_bytes < sizeof(fc_state_header)) return FC_ERR_INVALID;
  fc_state_header hd;
  std::memcpy(&hd, src, sizeof(hd));
  if (std::memcmp(hd.magic, FC_STATE_MAGIC, 8) != 0 || hd.version != 1) return FC_ERR_INVALID;
  if (hd.coeff_dtype != arc->coeff_dtype || hd.R != arc->R || hd.S != arc->S || hd.B != arc->B ||
      hd.H != arc->H || hd.D != arc->D)
    return FC_ERR_INVALID;
  if (hd.n_blocks < 0 || hd.tail_len < 0 || hd.tail_len >= hd.R) return FC_ERR_INVALID;
  if (hd.tail_len > 0) {
    if (!tail) return FC_ERR_INVALID;
    st = check_tail(tail, arc, false);
    if (st != FC_OK) return st;
    if (tail->dtype != hd.tail_dtype) return FC_ERR_INVALID;
  } else if (tail) {
    st = check_tail(tail, arc, true);
    if (st != FC_OK) return st;
  }
  const Parts p = parts_of(arc, hd.n_blocks, hd.tail_len, hd.tail_dtype);
  if (p.coeff != hd.coeff_bytes || p.scale != hd.scale_bytes || p.tail != hd.tail_bytes) return FC_ERR_INVALID;
  if (src_bytes < sizeof(hd) + size_t(p.coeff + p.scale + p.tail)) return FC_ERR_INVALID;
  if (hd.n_blocks > arc->capacity) return FC_ERR_CAPACITY;
  const uint8_t* in = static_cast<const uint8_t*>(src) + sizeof(hd);
  const int cesz = dtype_size(arc->coeff_dtype);
  for (int64_t b = 0; b < arc->B; ++b) {
    uint8_t* cd = static_cast<uint8_t*>(arc->coeffs) + b * arc->coeff_stride_b * cesz;
    st = copy_runs(cd, head_pitch(arc->coeff_stride_h, arc->H, size_t(p.coeff_row), cesz),
                   in + b * arc->H * p.coeff_row, size_t(p.coeff_row), size_t(p.coeff_row), size_t(arc->H),
                   cudaMemcpyHostToDevice, stream);
    if (st != FC_OK) return st;
    if (p.scale_row) {
      uint8_t* sd = reinterpret_cast<uint8_t*>(arc->scales) + b * arc->scale_stride_b * 4;
      st = copy_runs(sd, head_pitch(arc->scale_stride_h, arc->H, size_t(p.scale_row), 4),
                     in + p.coeff + b * arc->H * p.scale_row, size_t(p.scale_row), size_t(p.scale_row),
                     size_t(arc->H), cudaMemcpyHostToDevice, stream);
      if (st != FC_OK) return st;
    }
    if (p.tail_row) {
      const int tesz = dtype_size(tail->dtype);
      uint8_t* td = static_cast<uint8_t*>(tail->data) + b * tail->stride_b * tesz;
      st = copy_runs(td, head_pitch(tail->stride_h, arc->H, size_t(p.tail_row), tesz),
                     in + p.coeff + p.scale + b * arc->H * p.tail_row, size_t(p.tail_row), size_t(p.tail_row),
                     size_t(arc->H), cudaMemcpyHostToDevice, stream);
      if (st != FC_OK) return st;
    }
  }
  arc->n_blocks = hd.n_blocks;
  if (tail) tail->len = hd.tail_len;
  return FC_OK;
}
