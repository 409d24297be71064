// The block encoder shared by prefill compression, the single-token append and
// the fused decode step: C = M X for one block (the orthonormal DCT-II rows of
// flashcodec-kv README "Math"), kept frequencies only, accumulated in fp64,
// then int8 codes with one fp32 absmax/127 scale per (block, frequency) (README,
// quant_bits=8 paragraph; flashcodec/cache.py, _archive_spec) or rounded to the
// unquantised storage dtype. Every caller runs this same device code in the
// same order, so an archive built by any mix of them is bitwise the same.
#pragma once

#include <type_traits>

#include "fc_internal.cuh"

namespace fc {

struct StreamOut {
  void* coeffs;
  float* scales;
  int64_t cs_b, cs_h;  // coefficient element strides
  int64_t ss_b, ss_h;  // scale element strides
};

constexpr int kJC = 4;  // frequencies per pass over a block's rows

__device__ __forceinline__ double warp_max_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <int VEC>
__device__ __forceinline__ void store_codes(int8_t* p, const int (&code)[VEC]) {
  if constexpr (VEC == 1) {
    *p = static_cast<int8_t>(code[0]);
  } else if constexpr (VEC == 2) {
    const uint32_t w = (uint32_t(code[0]) & 0xffu) | ((uint32_t(code[1]) & 0xffu) << 8);
    *reinterpret_cast<unsigned short*>(p) = static_cast<unsigned short>(w);
  } else {
    uint32_t w[VEC / 4];
#pragma unroll
    for (int i = 0; i < VEC / 4; ++i) {
      w[i] = (uint32_t(code[4 * i]) & 0xffu) | ((uint32_t(code[4 * i + 1]) & 0xffu) << 8) |
             ((uint32_t(code[4 * i + 2]) & 0xffu) << 16) | ((uint32_t(code[4 * i + 3]) & 0xffu) << 24);
    }
    if constexpr (VEC == 4) {
      *reinterpret_cast<uint32_t*>(p) = w[0];
    } else {
      *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
    }
  }
}

template <typename T, int VEC>
__device__ __forceinline__ void store_row(T* p, const float (&x)[VEC]) {
  if constexpr (std::is_same_v<T, float>) {
    if constexpr (VEC % 4 == 0) {
#pragma unroll
      for (int i = 0; i < VEC / 4; ++i)
        reinterpret_cast<float4*>(p)[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
    } else if constexpr (VEC == 2) {
      *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
    } else {
      p[0] = x[0];
    }
  } else {
    static_assert(std::is_same_v<T, __nv_bfloat16>, "bf16 or f32 rows");
    if constexpr (VEC == 1) {
      p[0] = __float2bfloat16_rn(x[0]);
    } else {
      uint32_t w[VEC / 2];
#pragma unroll
      for (int i = 0; i < VEC / 2; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
      }
      if constexpr (VEC == 2) {
        *reinterpret_cast<uint32_t*>(p) = w[0];
      } else if constexpr (VEC == 4) {
        *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
      } else {
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

template <int VEC>
__device__ __forceinline__ void store_bf16_row(__nv_bfloat16* p, const __nv_bfloat16 (&h)[VEC]) {
  if constexpr (VEC == 1) {
    p[0] = h[0];
  } else {
    uint32_t w[VEC / 2];
#pragma unroll
    for (int i = 0; i < VEC / 2; ++i)
      w[i] = uint32_t(__bfloat16_as_ushort(h[2 * i])) | (uint32_t(__bfloat16_as_ushort(h[2 * i + 1])) << 16);
    if constexpr (VEC == 2) {
      *reinterpret_cast<uint32_t*>(p) = w[0];
    } else if constexpr (VEC == 4) {
      *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
    } else {
      *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// 1 / s for the quantiser (0 for s = 0) without an fp64 division: a
// single-precision seed refined by two Newton steps r <- r + r (1 - s r),
// accurate to about one fp64 ulp; scales outside the single-precision range
// divide. Every encoder runs this same sequence, so their codes agree
// bitwise; against the exact reciprocal a code can differ only where
// c / s lies within ~1e-13 of a half-integer.
__device__ __forceinline__ double quant_reciprocal(double s) {
  if (s == 0.0) return 0.0;
  if (!(s > 0x1p-120 && s < 0x1p120)) return 1.0 / s;
  double r = double(__frcp_rn(float(s)));
#pragma unroll
  for (int k = 0; k < 2; ++k) r = fma(r, fma(-s, r, 1.0), r);
  return r;
}

// Quantises (int8) or rounds (bf16 / f32) one coefficient row held in fp64
// and stores it at `row` (D elements; lane owns VEC) and, for int8, its scale.
template <typename TOut, int VEC>
__device__ __forceinline__ void store_coeff_row(const double (&c)[VEC], int lane, TOut* row,
                                                float* scl) {
  if constexpr (std::is_same_v<TOut, int8_t>) {
    double amax = 0.0;
#pragma unroll
    for (int v = 0; v < VEC; ++v) amax = fmax(amax, fabs(c[v]));
    amax = warp_max_d(amax);
    const double scale = amax * (1.0 / 127.0);  // within two ulps of amax / 127
    const double inv = quant_reciprocal(scale);
    int code[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) code[v] = max(-127, min(127, __double2int_rn(c[v] * inv)));
    store_codes<VEC>(row + lane * VEC, code);
    if (lane == 0) *scl = __double2float_rn(scale);
  } else if constexpr (std::is_same_v<TOut, float>) {
    float x[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) x[v] = __double2float_rn(c[v]);
    store_row<float, VEC>(row + lane * VEC, x);
  } else {
    // direct fp64 -> bf16 rounding, packed in pairs
    __nv_bfloat16 hb[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) hb[v] = __double2bfloat16(c[v]);
    store_bf16_row<VEC>(row + lane * VEC, hb);
  }
}

// Encodes the S kept frequencies of one block whose R token rows come from
// `row_at(t, xf)` (VEC floats of row t for this lane), kJC frequencies per
// pass, and stores them at `blk` (S x D elements) / `scl` (S floats).
// SC, RC > 0 fix S and R at compile time (the loops unroll, basis entries
// become constant operands and the frequency guards fold away); the
// arithmetic and its order are the same, so the codes are bitwise those of
// the runtime-sized form. For mirror-symmetric rows (the DCT with an even R:
// m[j][R-1-t] = (-1)^j m[j][t]) the sum runs over t < R/2 on
// u_t = x_t + x_{R-1-t} (even j) or w_t = x_t - x_{R-1-t} (odd j), formed in
// fp64: half the multiply-adds, the same value up to fp64 rounding.
template <typename TOut, int VEC, int SC = 0, int RC = 0, typename RowAt, typename BasisT>
__device__ __forceinline__ void encode_block(RowAt&& row_at, int R_, int S_, int D, int lane,
                                             const BasisT& basis, TOut* blk, float* scl) {
  const int R = RC > 0 ? RC : R_;
  const int S = SC > 0 ? SC : S_;
  const bool mirror = basis.mirror != 0;
  auto pass = [&](int j0) {
    double c[kJC][VEC];
#pragma unroll
    for (int jj = 0; jj < kJC; ++jj)
#pragma unroll
      for (int v = 0; v < VEC; ++v) c[jj][v] = 0.0;
    auto pair = [&](int t) {  // rows t and R-1-t folded (mirror rows)
      float xa[VEC], xb[VEC];
      row_at(t, xa);
      row_at(R - 1 - t, xb);
      double u[VEC], w[VEC];
#pragma unroll
      for (int v = 0; v < VEC; ++v) {
        const double da = double(xa[v]), db = double(xb[v]);
        u[v] = da + db;
        w[v] = da - db;
      }
#pragma unroll
      for (int jj = 0; jj < kJC; ++jj) {
        if (j0 + jj < S) {
          const double m = basis.m[j0 + jj][t];
#pragma unroll
          for (int v = 0; v < VEC; ++v) c[jj][v] = fma(m, ((j0 + jj) & 1) ? w[v] : u[v], c[jj][v]);
        }
      }
    };
    auto row = [&](int t) {
      float xf[VEC];
      row_at(t, xf);
      // one conversion per element (the conversion unit, not the fp64 FMAs,
      // bounds this loop otherwise)
      double xd[VEC];
#pragma unroll
      for (int v = 0; v < VEC; ++v) xd[v] = double(xf[v]);
#pragma unroll
      for (int jj = 0; jj < kJC; ++jj) {
        if (j0 + jj < S) {
          const double m = basis.m[j0 + jj][t];
#pragma unroll
          for (int v = 0; v < VEC; ++v) c[jj][v] = fma(m, xd[v], c[jj][v]);
        }
      }
    };
    if constexpr (RC > 0) {
      if (mirror) {
#pragma unroll
        for (int t = 0; t < RC / 2; ++t) pair(t);
      } else {
#pragma unroll
        for (int t = 0; t < RC; ++t) row(t);
      }
    } else if (mirror) {
#pragma unroll 2
      for (int t = 0; t < R / 2; ++t) pair(t);
    } else {
#pragma unroll 4
      for (int t = 0; t < R; ++t) row(t);
    }
#pragma unroll
    for (int jj = 0; jj < kJC; ++jj) {
      const int j = j0 + jj;
      if (j < S) store_coeff_row<TOut, VEC>(c[jj], lane, blk + int64_t(j) * D, scl ? scl + j : nullptr);
    }
  };
  if constexpr (SC > 0) {
#pragma unroll
    for (int j0 = 0; j0 < SC; j0 += kJC) pass(j0);
  } else {
    for (int j0 = 0; j0 < S; j0 += kJC) pass(j0);
  }
}


}  // namespace fc
