// Structural operations on one stream: the reconstructed view (block
// decompression X_hat = M^T C_hat plus the raw tail), exact crop, batch
// gather (flashcodec/cache.py, _CodecStream.read / _decode_pending, crop,
// select_batch). Declared in include/fc_view.h.
//
// The view kernel is a pure stream: per (b, h, block) it reads S rows of
// codes (and S scales) and writes R rows of D outputs, so HBM writes dominate
// (R*D*2 bytes of bf16 against S*D + 4*S bytes of int8 archive). One warp owns
// one (b, h, block) item at a time; lane l owns the D/32 consecutive columns
// [l*D/32, (l+1)*D/32), so every output row is one coalesced warp store and
// the S dequantised coefficient rows of those columns stay in registers.
#include <cuda_bf16.h>

#include <type_traits>

#include "fc_internal.cuh"
#include "fc_view.h"

namespace fc {
namespace {

constexpr int kViewThreads = 256;
constexpr int kViewWarps = kViewThreads / 32;

struct ViewArgs {
  const void* coeffs;
  const float* scales;  // null unless int8
  int64_t cs_b, cs_h;   // coefficient element strides
  int64_t ss_b, ss_h;   // scale strides
  const void* tail;     // null when no tail rows are copied
  int64_t ts_b, ts_h;   // tail element strides
  int32_t tail_dtype;
  int32_t tail_len;
  void* out;
  int64_t os_b, os_h, os_t;  // out element strides
  int64_t H;
  int64_t first;      // first decoded block
  int64_t count;      // decoded blocks per (b, h)
  int64_t out_row0;   // out row of token 0 of block `first`
  int64_t tail_row0;  // out row of tail token 0
  int32_t R, S;
  int32_t codec;      // FC_CODEC_DCT or FC_CODEC_PNG (decoding rows)
  int32_t rows;       // tokens t < rows of each block are written (<= R)
  int64_t block_items;  // B * H * count
  int64_t tail_items;   // B * H when tail rows are copied, else 0
};

// VEC consecutive outputs of one lane, rounded to the out dtype (bf16: round
// to nearest even, two values per conversion).
template <typename TO, int VEC>
__device__ __forceinline__ void store_out(TO* p, const float (&v)[VEC]) {
  if constexpr (std::is_same<TO, float>::value) {
    if constexpr (VEC == 1) {
      *p = v[0];
    } else if constexpr (VEC == 2) {
      *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
      for (int c = 0; c < VEC / 4; ++c)
        reinterpret_cast<float4*>(p)[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    }
  } else if constexpr (VEC == 1) {
    *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(v[0]);
  } else {
    uint32_t w[VEC / 2];
#pragma unroll
    for (int i = 0; i < VEC / 2; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
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

// The raw bytes of one lane's VEC consecutive coefficients of one frequency
// row, loaded ahead of their use and converted afterwards.
template <typename TC, int VEC>
struct RawRow {
  static constexpr int kBytes = VEC * int(sizeof(TC));
  static constexpr int kWords = kBytes >= 4 ? kBytes / 4 : 1;
  uint32_t w[kWords];

  __device__ __forceinline__ void load(const TC* p) {
    if constexpr (kBytes >= 16) {
#pragma unroll
      for (int c = 0; c < kBytes / 16; ++c) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + c);
        w[4 * c] = u.x;
        w[4 * c + 1] = u.y;
        w[4 * c + 2] = u.z;
        w[4 * c + 3] = u.w;
      }
    } else if constexpr (kBytes == 8) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
      w[0] = u.x;
      w[1] = u.y;
    } else if constexpr (kBytes == 4) {
      w[0] = __ldg(reinterpret_cast<const unsigned int*>(p));
    } else if constexpr (kBytes == 2) {
      w[0] = __ldg(reinterpret_cast<const unsigned short*>(p));
    } else {
      w[0] = static_cast<uint8_t>(__ldg(reinterpret_cast<const signed char*>(p)));
    }
  }

  // int8: exact, without a conversion instruction: the biased byte b + 128
  // becomes the low mantissa bits of 2^23, and 2^23 + 128 is subtracted.
  __device__ __forceinline__ void to_float(float (&out)[VEC]) const {
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      if constexpr (std::is_same<TC, int8_t>::value) {
        const uint32_t u = w[i / 4] ^ 0x80808080u;
        out[i] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7440u | uint32_t(i % 4))) - 8388736.0f;
      } else if constexpr (std::is_same<TC, __nv_bfloat16>::value) {
        const uint32_t x = w[i / 2];
        out[i] = __uint_as_float((i % 2) ? (x & 0xffff0000u) : (x << 16));
      } else {
        out[i] = __uint_as_float(w[i]);
      }
    }
  }
};

// Resident CTAs per SM the view kernel is compiled for, from the registers
// a lane holds: MAXS >= S coefficient rows of VEC values (and their raw
// prefetched words, twice as many for fp32 storage).
template <typename TC, int VEC, int MAXS>
constexpr int view_ctas_per_sm() {
  constexpr int held = MAXS * VEC * (sizeof(TC) == 4 ? 2 : 1);
  return held <= 16 ? 5 : held <= 32 ? 3 : held <= 64 ? 2 : 1;
}

// TC: stored coefficient type; TO: view dtype; VEC = D / 32. Loops over the
// frequencies j are unrolled to MAXS and guarded by j < S, so the rows are
// never indexed dynamically. Each warp walks its items with a stride of the
// grid's warp count and loads the next item's codes and scales before it
// writes the current item's R rows. Item counts fit in 31 bits (checked on
// the host).
template <typename TC, typename TO, int VEC, int MAXS>
__global__ void __launch_bounds__(kViewThreads, view_ctas_per_sm<TC, VEC, MAXS>())
    read_view_kernel(ViewArgs a, Basis basis) {
  __shared__ float m_s[kMaxS * kMaxR];  // m_s[j * R + t] = M[j][t]
  for (int i = threadIdx.x; i < a.S * a.R; i += kViewThreads) {
    const int j = i / a.R, t = i - j * a.R;
    m_s[i] = basis.m[j][t];
  }
  __syncthreads();

  constexpr int D = VEC * 32;
  constexpr bool kQuant = std::is_same<TC, int8_t>::value;
  const int lane = threadIdx.x & 31;
  const uint32_t warps = gridDim.x * kViewWarps;
  const uint32_t block_items = uint32_t(a.block_items);
  const uint32_t total = block_items + uint32_t(a.tail_items);
  const uint32_t count = uint32_t(a.count), H = uint32_t(a.H);

  RawRow<TC, VEC> raw[MAXS];
  float sc[MAXS];
  auto fetch = [&](uint32_t item) {
    const uint32_t bh = item / count;
    const int64_t n = a.first + (item - bh * count);
    const uint32_t b = bh / H, h = bh - b * H;
    const TC* cp = static_cast<const TC*>(a.coeffs) + b * a.cs_b + h * a.cs_h + n * a.S * D + lane * VEC;
    const float* sp = kQuant ? a.scales + b * a.ss_b + h * a.ss_h + n * a.S : nullptr;
#pragma unroll
    for (int j = 0; j < MAXS; ++j) {
      if (j < a.S) {
        raw[j].load(cp + j * D);
        if constexpr (kQuant) sc[j] = __ldg(sp + j);
      }
    }
  };

  uint32_t item = blockIdx.x * kViewWarps + (threadIdx.x >> 5);
  if (item < block_items) fetch(item);
  for (; item < total; item += warps) {
    if (item < block_items) {
      float c[MAXS][VEC];
#pragma unroll
      for (int j = 0; j < MAXS; ++j) {
        if (j < a.S) {
          raw[j].to_float(c[j]);
          if constexpr (kQuant) {
#pragma unroll
            for (int v = 0; v < VEC; ++v) c[j][v] *= sc[j];
          }
        }
      }
      const uint32_t bh = item / count;
      const int64_t nr = item - bh * count;  // block index relative to `first`
      const uint32_t b = bh / H, h = bh - b * H;
      if (item + warps < block_items) fetch(item + warps);
      TO* op = static_cast<TO*>(a.out) + b * a.os_b + h * a.os_h + (a.out_row0 + nr * a.R) * a.os_t +
               lane * VEC;
      for (int t = 0; t < a.rows; ++t) {
        float x[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) x[v] = 0.f;
#pragma unroll
        for (int j = 0; j < MAXS; ++j) {
          if (j < a.S) {
            const float mj = m_s[j * a.R + t];
#pragma unroll
            for (int v = 0; v < VEC; ++v) x[v] = fmaf(mj, c[j][v], x[v]);
          }
        }
        store_out<TO, VEC>(op + t * a.os_t, x);
      }
    } else {
      // raw tail rows, converted to the view dtype
      const uint32_t bh = item - block_items;
      const uint32_t b = bh / H, h = bh - b * H;
      TO* op = static_cast<TO*>(a.out) + b * a.os_b + h * a.os_h + a.tail_row0 * a.os_t + lane * VEC;
      const int64_t tbase = b * a.ts_b + h * a.ts_h + lane * VEC;
      for (int r = 0; r < a.tail_len; ++r) {
        float x[VEC];
#pragma unroll
        for (int v = 0; v < VEC; ++v) x[v] = load_any(a.tail, tbase + int64_t(r) * D + v, a.tail_dtype);
        store_out<TO, VEC>(op + r * a.os_t, x);
      }
    }
  }
}

// The view of an int8 archive in the common geometry (D = 128, R = 8 or 16,
// whole blocks, output rows contiguous: row stride D) with S and R fixed at
// compile time. The row loop is unrolled, so every basis entry M[j][t] is an
// FMA operand at a fixed offset of the kernel's parameters and every store
// an immediate offset from the item's output pointer. Warp w takes the
// contiguous item range [w * per, (w + 1) * per) and walks (b, h, block) by
// counters (no divisions inside the loop), loading the next block's codes
// and scales before it writes the current block's R rows; the first B * H
// warps also copy one (b, h) raw tail each.
template <int S>
constexpr int view_rows_ctas_per_sm() {
  return S >= 4 ? 3 : 4;  // registers: S coefficient rows of 4 values besides the output rows
}

template <typename TO, int S, int R>
__global__ void __launch_bounds__(kViewThreads, view_rows_ctas_per_sm<S>())
    read_view_rows_kernel(ViewArgs a, Basis basis) {
  constexpr int VEC = 4, D = 128;
  const int lane = threadIdx.x & 31;
  const uint32_t nw = gridDim.x * kViewWarps;
  const uint32_t gw = blockIdx.x * kViewWarps + (threadIdx.x >> 5);
  const uint32_t H = uint32_t(a.H), count = uint32_t(a.count);
  if (gw < uint32_t(a.tail_items)) {
    const uint32_t b = gw / H, h = gw - b * H;
    TO* op = static_cast<TO*>(a.out) + b * a.os_b + h * a.os_h + a.tail_row0 * D + lane * VEC;
    const int64_t tbase = b * a.ts_b + h * a.ts_h + lane * VEC;
    for (int r = 0; r < a.tail_len; ++r) {
      float x[VEC];
#pragma unroll
      for (int v = 0; v < VEC; ++v) x[v] = load_any(a.tail, tbase + int64_t(r) * D + v, a.tail_dtype);
      store_out<TO, VEC>(op + r * D, x);
    }
  }
  const uint32_t items = uint32_t(a.block_items);
  const uint32_t per = (items + nw - 1) / nw;
  uint32_t i = gw * per;
  const uint32_t iend = min(i + per, items);
  if (i >= iend) return;
  uint32_t bh = i / count;
  uint32_t n = i - bh * count;
  uint32_t b = bh / H, h = bh - b * H;
  const int8_t* cp;
  const float* sp;
  TO* op;
  auto locate = [&]() {
    const int64_t blk = a.first + n;
    cp = static_cast<const int8_t*>(a.coeffs) + b * a.cs_b + h * a.cs_h + blk * (S * D) + lane * VEC;
    sp = a.scales + b * a.ss_b + h * a.ss_h + blk * S;
    op = static_cast<TO*>(a.out) + b * a.os_b + h * a.os_h + (a.out_row0 + int64_t(n) * R) * D + lane * VEC;
  };
  locate();
  RawRow<int8_t, VEC> raw[S];
  float sc[S];
#pragma unroll
  for (int j = 0; j < S; ++j) {
    raw[j].load(cp + j * D);
    sc[j] = __ldg(sp + j);
  }
  for (; i < iend; ++i) {
    float c[S][VEC];
#pragma unroll
    for (int j = 0; j < S; ++j) {
      raw[j].to_float(c[j]);
#pragma unroll
      for (int v = 0; v < VEC; ++v) c[j][v] *= sc[j];
    }
    TO* o = op;
    if (i + 1 < iend) {
      if (++n == count) {
        n = 0;
        if (++h == H) {
          h = 0;
          ++b;
        }
        locate();
      } else {
        cp += S * D;
        sp += S;
        op += R * D;
      }
#pragma unroll
      for (int j = 0; j < S; ++j) {
        raw[j].load(cp + j * D);
        sc[j] = __ldg(sp + j);
      }
    }
#pragma unroll
    for (int t = 0; t < R; ++t) {
      float x[VEC];
#pragma unroll
      for (int v = 0; v < VEC; ++v) x[v] = basis.m[0][t] * c[0][v];
#pragma unroll
      for (int j = 1; j < S; ++j)
#pragma unroll
        for (int v = 0; v < VEC; ++v) x[v] = fmaf(basis.m[j][t], c[j][v], x[v]);
      store_out<TO, VEC>(o + t * D, x);
    }
  }
}

// ------------------------------------------------------------- batch gather

struct GatherIndex {
  int32_t src_b[FC_SELECT_MAX_BATCH];
};

struct GatherArgs {
  const uint8_t* src_c;
  uint8_t* dst_c;
  int64_t src_cb, src_ch, dst_cb, dst_ch;  // bytes
  int64_t c_bytes;                         // live coefficient bytes per (b, h)
  const uint8_t* src_s;
  uint8_t* dst_s;
  int64_t src_sb, src_sh, dst_sb, dst_sh;  // bytes
  int64_t s_words;                         // live scale floats per (b, h)
  const uint8_t* src_t;
  uint8_t* dst_t;
  int64_t src_tb, src_th, dst_tb, dst_th;  // bytes
  int64_t t_bytes;                         // live tail bytes per (b, h)
  int64_t H;
};

// blockIdx.y = destination (b, h) pair; blockIdx.x strides over its bytes.
// Coefficient and tail segments are multiples of 16 bytes at 16-byte aligned
// addresses (D * element size >= 32 bytes per row; strides are validated
// multiples of 16 bytes); scales are copied as 4-byte words.
__global__ void __launch_bounds__(256) select_batch_kernel(GatherArgs a, GatherIndex idx) {
  const int64_t bh = blockIdx.y;
  const int64_t b = bh / a.H, h = bh - b * a.H;
  const int64_t sb = idx.src_b[b];
  const int64_t step = int64_t(gridDim.x) * blockDim.x;
  const int64_t i0 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  {
    const uint4* s = reinterpret_cast<const uint4*>(a.src_c + sb * a.src_cb + h * a.src_ch);
    uint4* d = reinterpret_cast<uint4*>(a.dst_c + b * a.dst_cb + h * a.dst_ch);
    for (int64_t i = i0; i < a.c_bytes / 16; i += step) d[i] = s[i];
  }
  if (a.src_s) {
    const float* s = reinterpret_cast<const float*>(a.src_s + sb * a.src_sb + h * a.src_sh);
    float* d = reinterpret_cast<float*>(a.dst_s + b * a.dst_sb + h * a.dst_sh);
    for (int64_t i = i0; i < a.s_words; i += step) d[i] = s[i];
  }
  if (a.src_t) {
    const uint4* s = reinterpret_cast<const uint4*>(a.src_t + sb * a.src_tb + h * a.src_th);
    uint4* d = reinterpret_cast<uint4*>(a.dst_t + b * a.dst_tb + h * a.dst_th);
    for (int64_t i = i0; i < a.t_bytes / 16; i += step) d[i] = s[i];
  }
}

// ------------------------------------------------------------------- host

template <typename F>
int dispatch_coeff(int dt, F&& f) {
  if (dt == FC_DTYPE_I8) return f(int8_t{});
  if (dt == FC_DTYPE_BF16) return f(__nv_bfloat16{});
  if (dt == FC_DTYPE_F32) return f(float{});
  return FC_ERR_UNSUPPORTED;
}

template <typename F>
int dispatch_view(int dt, F&& f) {
  if (dt == FC_DTYPE_BF16) return f(__nv_bfloat16{});
  if (dt == FC_DTYPE_F32) return f(float{});
  return FC_ERR_INVALID;
}

template <typename F>
int dispatch_d(int64_t D, F&& f) {
  switch (D) {
    case 32: return f(std::integral_constant<int, 1>{});
    case 64: return f(std::integral_constant<int, 2>{});
    case 128: return f(std::integral_constant<int, 4>{});
    case 256: return f(std::integral_constant<int, 8>{});
    default: return FC_ERR_UNSUPPORTED;
  }
}

template <typename TC, typename TO, int VEC, int MAXS>
int launch_view_as(const ViewArgs& a, const Basis& basis, int64_t total, fc_stream stream) {
  int64_t grid = (total + kViewWarps - 1) / kViewWarps;
  const int64_t cap = int64_t(sm_count()) * view_ctas_per_sm<TC, VEC, MAXS>();
  if (grid > cap) grid = cap;
  read_view_kernel<TC, TO, VEC, MAXS><<<unsigned(grid), kViewThreads, 0, stream>>>(a, basis);
  return cuda_status(cudaGetLastError());
}

// Launches the view kernel for `a` (items already counted). Grid: enough
// warps for every item, at most one wave of resident CTAs (a grid-stride
// loop covers the rest).
template <typename TO, int S, int R>
int launch_view_rows(const ViewArgs& a, const Basis& basis, int64_t total, fc_stream stream) {
  int64_t grid = (total + kViewWarps - 1) / kViewWarps;
  const int64_t cap = int64_t(sm_count()) * view_rows_ctas_per_sm<S>();
  if (grid > cap) grid = cap;
  read_view_rows_kernel<TO, S, R><<<unsigned(grid), kViewThreads, 0, stream>>>(a, basis);
  return cuda_status(cudaGetLastError());
}

// the unrolled kernel for int8, D = 128, whole blocks of R = 8 or 16 and
// contiguous output rows; FC_ERR_UNSUPPORTED (nothing launched) otherwise
template <typename TO>
int try_view_rows(const ViewArgs& a, const Basis& basis, int64_t total, fc_stream stream) {
  if (a.rows != a.R || a.os_t != 128) return FC_ERR_UNSUPPORTED;
  if (a.tail_items && a.tail_len > a.R) return FC_ERR_UNSUPPORTED;
  if (a.R == 8) {
    switch (a.S) {
      case 1: return launch_view_rows<TO, 1, 8>(a, basis, total, stream);
      case 2: return launch_view_rows<TO, 2, 8>(a, basis, total, stream);
      case 3: return launch_view_rows<TO, 3, 8>(a, basis, total, stream);
      case 4: return launch_view_rows<TO, 4, 8>(a, basis, total, stream);
      default: break;
    }
  } else if (a.R == 16) {
    switch (a.S) {
      case 2: return launch_view_rows<TO, 2, 16>(a, basis, total, stream);
      case 4: return launch_view_rows<TO, 4, 16>(a, basis, total, stream);
      case 8: return launch_view_rows<TO, 8, 16>(a, basis, total, stream);
      default: break;
    }
  }
  return FC_ERR_UNSUPPORTED;
}

int launch_view(const ViewArgs& a, int coeff_dtype, int out_dtype, int64_t D, fc_stream stream) {
  const int64_t total = a.block_items + a.tail_items;
  if (total == 0) return FC_OK;
  if (total >= (int64_t(1) << 31)) return FC_ERR_UNSUPPORTED;
  Basis basis;
  make_basis(a.codec, a.R, a.S, &basis);
  if (coeff_dtype == FC_DTYPE_I8 && D == 128) {
    const int st = out_dtype == FC_DTYPE_BF16 ? try_view_rows<__nv_bfloat16>(a, basis, total, stream)
                   : out_dtype == FC_DTYPE_F32 ? try_view_rows<float>(a, basis, total, stream)
                                               : FC_ERR_UNSUPPORTED;
    if (st != FC_ERR_UNSUPPORTED) return st;
  }
  return dispatch_coeff(coeff_dtype, [&](auto tc) {
    using TC = decltype(tc);
    return dispatch_view(out_dtype, [&](auto to) {
      using TO = decltype(to);
      return dispatch_d(D, [&](auto vec) {
        constexpr int VEC = decltype(vec)::value;
        if (a.S <= 2) return launch_view_as<TC, TO, VEC, 2>(a, basis, total, stream);
        if (a.S <= 4) return launch_view_as<TC, TO, VEC, 4>(a, basis, total, stream);
        if (a.S <= 8) return launch_view_as<TC, TO, VEC, 8>(a, basis, total, stream);
        return launch_view_as<TC, TO, VEC, kMaxS>(a, basis, total, stream);
      });
    });
  });
}

void fill_archive_side(ViewArgs& a, const fc_archive* arc) {
  a.coeffs = arc->coeffs;
  a.scales = arc->coeff_dtype == FC_DTYPE_I8 ? arc->scales : nullptr;
  a.cs_b = arc->coeff_stride_b;
  a.cs_h = arc->coeff_stride_h;
  a.ss_b = arc->scale_stride_b;
  a.ss_h = arc->scale_stride_h;
  a.H = arc->H;
  a.R = arc->R;
  a.S = arc->S;
  a.codec = arc->codec;
}

// [lo, hi) byte span of every element a (B, H, extent) tensor can address.
struct Span {
  uintptr_t lo, hi;
};
Span span_of(const void* p, int64_t B, int64_t H, int64_t sb, int64_t sh, int64_t extent, int64_t esz) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return {lo, lo + uintptr_t(((B - 1) * sb + (H - 1) * sh + extent) * esz)};
}
bool overlap(Span x, Span y) { return x.lo < y.hi && y.lo < x.hi; }

}  // namespace
}  // namespace fc

using namespace fc;

extern "C" int fc_read_view(const fc_archive* arc, const fc_tail* tail, int64_t first_block, void* out,
                            int32_t out_dtype, const int64_t* out_strides, int64_t out_tokens,
                            fc_stream stream) {
  int st = check_archive(arc);
  if (st != FC_OK) return st;
  if (tail && (st = check_tail(tail, arc, true)) != FC_OK) return st;
  const int64_t len = tail ? tail->len : 0;
  if (first_block < 0 || first_block > arc->n_blocks) return FC_ERR_INVALID;
  if (out_dtype != FC_DTYPE_BF16 && out_dtype != FC_DTYPE_F32) return FC_ERR_INVALID;
  if (!out || !aligned16(out) || !out_strides || out_strides[3] != 1) return FC_ERR_INVALID;
  const int64_t esz = dtype_size(out_dtype);
  for (int i = 0; i < 3; ++i)
    if (out_strides[i] < 0 || (out_strides[i] * esz) % 16) return FC_ERR_INVALID;
  const int64_t rows = arc->n_blocks * arc->R + len;
  if (out_tokens < rows) return FC_ERR_INVALID;
  // rows, heads and batches of `out` must not alias one another
  if (out_tokens > 1 && out_strides[2] < arc->D) return FC_ERR_INVALID;
  if (arc->H > 1 && out_strides[1] < out_tokens * out_strides[2]) return FC_ERR_INVALID;
  if (arc->B > 1 && out_strides[0] < arc->H * out_strides[1]) return FC_ERR_INVALID;

  ViewArgs a{};
  fill_archive_side(a, arc);
  a.out = out;
  a.os_b = out_strides[0];
  a.os_h = out_strides[1];
  a.os_t = out_strides[2];
  a.first = first_block;
  a.count = arc->n_blocks - first_block;
  a.out_row0 = first_block * arc->R;
  a.rows = arc->R;
  a.block_items = arc->B * arc->H * a.count;
  a.tail = len > 0 ? tail->data : nullptr;
  a.tail_dtype = tail ? tail->dtype : FC_DTYPE_F32;
  a.tail_len = int32_t(len);
  a.ts_b = tail ? tail->stride_b : 0;
  a.ts_h = tail ? tail->stride_h : 0;
  a.tail_row0 = arc->n_blocks * arc->R;
  a.tail_items = len > 0 ? arc->B * arc->H : 0;
  return launch_view(a, arc->coeff_dtype, out_dtype, arc->D, stream);
}

extern "C" int fc_crop(fc_archive* arc, fc_tail* tail, int64_t tokens_to_remove, fc_stream stream) {
  int st = check_archive(arc);
  if (st != FC_OK) return st;
  if (!tail) return FC_ERR_INVALID;
  if ((st = check_tail(tail, arc, true)) != FC_OK) return st;
  if (tokens_to_remove > 0) return FC_ERR_INVALID;
  if (tokens_to_remove == 0) return FC_OK;
  const int64_t len = arc->n_blocks * arc->R + tail->len;
  const int64_t remove = -tokens_to_remove;
  const int64_t keep = remove >= len ? 0 : len - remove;
  const int64_t kb = keep / arc->R, rest = keep - kb * arc->R;
  if (kb < arc->n_blocks && rest > 0) {
    if (!tail->data) return FC_ERR_INVALID;
    // block kb, tokens [0, rest), decoded into tail rows [0, rest)
    ViewArgs a{};
    fill_archive_side(a, arc);
    a.out = tail->data;
    a.os_b = tail->stride_b;
    a.os_h = tail->stride_h;
    a.os_t = arc->D;
    a.first = kb;
    a.count = 1;
    a.out_row0 = 0;
    a.rows = int32_t(rest);
    a.block_items = arc->B * arc->H;
    a.tail = nullptr;
    a.tail_items = 0;
    st = launch_view(a, arc->coeff_dtype, tail->dtype, arc->D, stream);
    if (st != FC_OK) return st;
  }
  if (kb < arc->n_blocks) arc->n_blocks = kb;
  tail->len = int32_t(rest);
  return FC_OK;
}

extern "C" int fc_select_batch(const fc_archive* src, const fc_tail* src_tail, const int64_t* idx,
                               int64_t n_idx, fc_archive* dst, fc_tail* dst_tail, fc_stream stream) {
  int st = check_archive(src);
  if (st != FC_OK) return st;
  if ((st = check_archive(dst)) != FC_OK) return st;
  if (!idx || n_idx < 1) return FC_ERR_INVALID;
  if (n_idx > FC_SELECT_MAX_BATCH) return FC_ERR_UNSUPPORTED;
  if (dst->B != n_idx || dst->H != src->H || dst->R != src->R || dst->S != src->S || dst->D != src->D ||
      dst->coeff_dtype != src->coeff_dtype)
    return FC_ERR_INVALID;
  if (dst->capacity < src->n_blocks) return FC_ERR_CAPACITY;
  if ((src_tail == nullptr) != (dst_tail == nullptr)) return FC_ERR_INVALID;
  if (src_tail) {
    if ((st = check_tail(src_tail, src, true)) != FC_OK) return st;
    if ((st = check_tail(dst_tail, dst, src_tail->len == 0)) != FC_OK) return st;
    if (dst_tail->dtype != src_tail->dtype) return FC_ERR_INVALID;
  }
  GatherIndex gi;
  for (int64_t i = 0; i < n_idx; ++i) {
    if (idx[i] < 0 || idx[i] >= src->B) return FC_ERR_INVALID;
    gi.src_b[i] = int32_t(idx[i]);
  }
  const int64_t esz = dtype_size(src->coeff_dtype);
  const int64_t per_head = src->S * src->D;
  // source and destination must be disjoint (the copy is not ordered)
  if (overlap(span_of(src->coeffs, src->B, src->H, src->coeff_stride_b, src->coeff_stride_h,
                      src->capacity * per_head, esz),
              span_of(dst->coeffs, dst->B, dst->H, dst->coeff_stride_b, dst->coeff_stride_h,
                      dst->capacity * per_head, esz)))
    return FC_ERR_INVALID;
  if (src->scales &&
      overlap(span_of(src->scales, src->B, src->H, src->scale_stride_b, src->scale_stride_h,
                      src->capacity * src->S, 4),
              span_of(dst->scales, dst->B, dst->H, dst->scale_stride_b, dst->scale_stride_h,
                      dst->capacity * dst->S, 4)))
    return FC_ERR_INVALID;
  const bool copy_tail = src_tail && src_tail->len > 0;
  const int64_t tesz = src_tail ? dtype_size(src_tail->dtype) : 0;
  if (copy_tail &&
      overlap(span_of(src_tail->data, src->B, src->H, src_tail->stride_b, src_tail->stride_h,
                      int64_t(src->R) * src->D, tesz),
              span_of(dst_tail->data, dst->B, dst->H, dst_tail->stride_b, dst_tail->stride_h,
                      int64_t(dst->R) * dst->D, tesz)))
    return FC_ERR_INVALID;
  const int64_t pairs = n_idx * src->H;
  if (pairs > 65535) return FC_ERR_UNSUPPORTED;

  GatherArgs a{};
  a.src_c = static_cast<const uint8_t*>(src->coeffs);
  a.dst_c = static_cast<uint8_t*>(dst->coeffs);
  a.src_cb = src->coeff_stride_b * esz;
  a.src_ch = src->coeff_stride_h * esz;
  a.dst_cb = dst->coeff_stride_b * esz;
  a.dst_ch = dst->coeff_stride_h * esz;
  a.c_bytes = src->n_blocks * per_head * esz;
  if (src->scales) {
    a.src_s = reinterpret_cast<const uint8_t*>(src->scales);
    a.dst_s = reinterpret_cast<uint8_t*>(dst->scales);
    a.src_sb = src->scale_stride_b * 4;
    a.src_sh = src->scale_stride_h * 4;
    a.dst_sb = dst->scale_stride_b * 4;
    a.dst_sh = dst->scale_stride_h * 4;
    a.s_words = src->n_blocks * src->S;
  }
  if (copy_tail) {
    a.src_t = static_cast<const uint8_t*>(src_tail->data);
    a.dst_t = static_cast<uint8_t*>(dst_tail->data);
    a.src_tb = src_tail->stride_b * tesz;
    a.src_th = src_tail->stride_h * tesz;
    a.dst_tb = dst_tail->stride_b * tesz;
    a.dst_th = dst_tail->stride_h * tesz;
    a.t_bytes = int64_t(src_tail->len) * src->D * tesz;
  }
  a.H = src->H;
  const int64_t work = a.c_bytes / 16 > a.t_bytes / 16 ? a.c_bytes / 16 : a.t_bytes / 16;
  const int64_t most = work > a.s_words ? work : a.s_words;
  if (most > 0) {
    int64_t gx = (most + 255) / 256;
    if (gx > 1024) gx = 1024;
    select_batch_kernel<<<dim3(unsigned(gx), unsigned(pairs)), 256, 0, stream>>>(a, gi);
    if ((st = cuda_status(cudaGetLastError())) != FC_OK) return st;
  }
  dst->n_blocks = src->n_blocks;
  if (dst_tail) dst_tail->len = src_tail->len;
  return FC_OK;
}
