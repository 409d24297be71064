// Internal helpers shared by the libfc translation units (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fc.h"

namespace fc {

constexpr int kMaxR = 32;  // tokens per block
constexpr int kMaxS = 16;  // kept frequencies
constexpr int kMaxD = 256;

// Encoder rows M[j][t] of the orthonormal DCT-II in fp32 (flashcodec-kv README,
// "Math"); passed by value as a kernel parameter.
struct Basis {
  float m[kMaxS][kMaxR];
};

// Host: the decoding rows of the codec in fp32: for the DCT,
// M[j][t] = c_j cos(pi / R (t + 1/2) j) in double, rounded to fp32; for the
// PNG tier, m[j][t] = 1 for j <= t (cumulative sum).
void make_basis(int codec, int R, int S, Basis* out);

// The same rows in double precision (used by the compression kernels, which
// take the quantiser's rounding decision in fp64).
struct BasisF64 {
  double m[kMaxS][kMaxR];
  // 1 when row j is (-1)^j-symmetric, m[j][R-1-t] = (-1)^j m[j][t] (the DCT
  // with an even R): the encoder then folds the mirror rows first
  int32_t mirror;
};
// Host: the encoding rows of the codec in fp64 (the DCT rows; for the PNG
// tier the anchor row and the first differences).
void make_basis_f64(int codec, int R, int S, BasisF64* out);

// Host: SM count of the current device (cached per device).
int sm_count();

inline int dtype_size(int dt) {
  return dt == FC_DTYPE_F32 ? 4 : dt == FC_DTYPE_BF16 ? 2 : dt == FC_DTYPE_I8 ? 1 : 0;
}

inline bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// Host validation of one archive descriptor (shape, dtype, alignment).
int check_archive(const fc_archive* a);
// Host validation of a tail descriptor against its archive.
int check_tail(const fc_tail* t, const fc_archive* a, bool allow_null_data);

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? FC_OK : FC_ERR_CUDA; }

// Workspace layout (bytes): [status 256][tickets B*Hq*4, padded to 256]
// [m B*Hq*ns*4 pad][l B*Hq*ns*4 pad][acc B*Hq*ns*D*4].
struct WorkspaceLayout {
  size_t status, tickets, m, l, acc, total;
};
inline size_t pad256(size_t x) { return (x + 255) & ~size_t(255); }
inline WorkspaceLayout workspace_layout(int64_t B, int64_t Hq, int64_t D, int64_t ns) {
  WorkspaceLayout w;
  const size_t rows = size_t(B) * size_t(Hq) * size_t(ns);
  w.status = 0;
  w.tickets = 256;
  w.m = w.tickets + pad256(size_t(B) * size_t(Hq) * 4);
  w.l = w.m + pad256(rows * 4);
  w.acc = w.l + pad256(rows * 4);
  w.total = w.acc + pad256(rows * size_t(D) * 4);
  return w;
}

// ------------------------------------------------------------------ device

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Unpacks one 32-bit word holding 4 / sizeof(T) elements into floats.
template <typename T>
__device__ __forceinline__ void unpack_word(uint32_t w, float* out);
template <>
__device__ __forceinline__ void unpack_word<int8_t>(uint32_t w, float* out) {
#pragma unroll
  for (int i = 0; i < 4; ++i) out[i] = static_cast<float>(static_cast<int8_t>(w >> (8 * i)));
}
template <>
__device__ __forceinline__ void unpack_word<__nv_bfloat16>(uint32_t w, float* out) {
  out[0] = __uint_as_float(w << 16);
  out[1] = __uint_as_float(w & 0xffff0000u);
}
template <>
__device__ __forceinline__ void unpack_word<float>(uint32_t w, float* out) {
  out[0] = __uint_as_float(w);
}

// Loads VEC consecutive elements (aligned to VEC * sizeof(T) bytes) as floats.
template <typename T, int VEC>
__device__ __forceinline__ void load_vec(const T* __restrict__ p, float (&out)[VEC]) {
  constexpr int kBytes = VEC * int(sizeof(T));
  constexpr int kPerWord = 4 / int(sizeof(T));
  if constexpr (kBytes >= 16) {
#pragma unroll
    for (int c = 0; c < kBytes / 16; ++c) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + c);
      unpack_word<T>(u.x, &out[c * 4 * kPerWord + 0 * kPerWord]);
      unpack_word<T>(u.y, &out[c * 4 * kPerWord + 1 * kPerWord]);
      unpack_word<T>(u.z, &out[c * 4 * kPerWord + 2 * kPerWord]);
      unpack_word<T>(u.w, &out[c * 4 * kPerWord + 3 * kPerWord]);
    }
  } else if constexpr (kBytes == 8) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    unpack_word<T>(u.x, &out[0]);
    unpack_word<T>(u.y, &out[kPerWord]);
  } else if constexpr (kBytes == 4) {
    unpack_word<T>(__ldg(reinterpret_cast<const unsigned int*>(p)), &out[0]);
  } else if constexpr (kBytes == 2) {
    const uint32_t w = __ldg(reinterpret_cast<const unsigned short*>(p));
    if constexpr (sizeof(T) == 1) {
      out[0] = static_cast<float>(static_cast<int8_t>(w));
      out[1] = static_cast<float>(static_cast<int8_t>(w >> 8));
    } else {
      out[0] = __uint_as_float(w << 16);
    }
  } else {
    out[0] = static_cast<float>(static_cast<int8_t>(__ldg(reinterpret_cast<const signed char*>(p))));
  }
}

// Loads one element of a runtime dtype (FC_DTYPE_F32 or FC_DTYPE_BF16) as float.
__device__ __forceinline__ float load_any(const void* p, int64_t idx, int dtype) {
  if (dtype == FC_DTYPE_F32) return __ldg(static_cast<const float*>(p) + idx);
  const unsigned short h = __ldg(static_cast<const unsigned short*>(p) + idx);
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

}  // namespace fc
