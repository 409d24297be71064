// Block-DCT codec kernels: prefill compression, single-token append and the
// archive's growth copy.
//
// flashcodec-kv README "Math": a block X (R x D) is encoded as C = M X with the
// orthonormal DCT-II rows M; the S lowest frequencies are kept. With int8
// storage each (block, frequency) row keeps one fp32 scale over D
// (README, quant_bits=8 paragraph; flashcodec/cache.py, _archive_spec):
// scale = max_d |C| / 127 and code = clamp(rint(C / scale), -127, 127), an
// all-zero row storing scale 0 and codes 0. Only complete blocks are archived
// (flashcodec/cache.py, _CodecStream.append).
//
// Work mapping: one warp per (b, h, block); lane l owns the VEC = D / 32
// consecutive channels [l * VEC, (l + 1) * VEC), so every token row is one
// coalesced warp-wide load and every coefficient row one coalesced store. The
// coefficients accumulate in registers in fp64 (t ascending, fused
// multiply-add, four frequencies per pass over the block's rows), the absmax
// is a warp-shuffle max, and the quantiser takes its rounding decision in fp64
// (round-to-nearest-even of C times the reciprocal scale), so codes agree with
// an fp64 evaluation of the definition except where C / scale lies within a
// few fp64 ulps of a half-integer; unquantised coefficients are rounded from
// fp64 straight to the storage dtype. The fp64 work stays below the HBM
// stream's time on sm_100a. Compression of a prefill and of an appended block
// run the same device code in the same order, so an archive built token by
// token is bitwise identical to one built in a single call.
#include <type_traits>

#include "fc_encode.cuh"

namespace fc {
namespace {

struct CompressArgs {
  const void* x;
  int64_t xs_b, xs_h, xs_t;
  int B, H, R, S, D;
  int64_t n_full, slot0;
  StreamOut out;
  void* tail;  // may be null
  int64_t ts_b, ts_h;
  int n_rem;
};

template <int VEC, typename TIn, typename TOut>
__global__ void __launch_bounds__(256) compress_blocks_kernel(CompressArgs a, BasisF64 basis) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_items = int64_t(a.B) * a.H * a.n_full;
  const TIn* x = static_cast<const TIn*>(a.x);
  if (w < n_items) {
    const int64_t n = w % a.n_full;
    const int64_t bh = w / a.n_full;
    const int h = int(bh % a.H), b = int(bh / a.H);
    const TIn* src = x + b * a.xs_b + h * a.xs_h + n * a.R * a.xs_t + lane * VEC;
    TOut* blk = static_cast<TOut*>(a.out.coeffs) + b * a.out.cs_b + h * a.out.cs_h +
                (a.slot0 + n) * a.S * a.D;
    float* scl = a.out.scales ? a.out.scales + b * a.out.ss_b + h * a.out.ss_h + (a.slot0 + n) * a.S
                              : nullptr;
    encode_block<TOut, VEC>([&](int t, float (&xf)[VEC]) { load_vec<TIn, VEC>(src + t * a.xs_t, xf); },
                            a.R, a.S, a.D, lane, basis, blk, scl);
  } else if (a.tail != nullptr && w < n_items + int64_t(a.B) * a.H) {
    // copy the T mod R remaining tokens of (b, h) into its raw tail rows
    const int64_t bh = w - n_items;
    const int h = int(bh % a.H), b = int(bh / a.H);
    const TIn* src = x + b * a.xs_b + h * a.xs_h + a.n_full * a.R * a.xs_t + lane * VEC;
    TIn* dst = static_cast<TIn*>(a.tail) + b * a.ts_b + h * a.ts_h + lane * VEC;
    for (int i = 0; i < a.n_rem; ++i) {
      float xv[VEC];
      load_vec<TIn, VEC>(src + i * a.xs_t, xv);
      store_row<TIn, VEC>(dst + int64_t(i) * a.D, xv);
    }
  }
}

// As load_vec, from memory this thread may also write (shared memory): plain
// loads instead of the read-only path.
template <typename T, int VEC>
__device__ __forceinline__ void load_vec_plain(const T* p, float (&out)[VEC]) {
  constexpr int kBytes = VEC * int(sizeof(T));
  constexpr int kPerWord = 4 / int(sizeof(T));
  static_assert(kBytes >= 4, "at least one word");
  if constexpr (kBytes >= 16) {
#pragma unroll
    for (int c = 0; c < kBytes / 16; ++c) {
      const uint4 u = reinterpret_cast<const uint4*>(p)[c];
      unpack_word<T>(u.x, &out[c * 4 * kPerWord + 0 * kPerWord]);
      unpack_word<T>(u.y, &out[c * 4 * kPerWord + 1 * kPerWord]);
      unpack_word<T>(u.z, &out[c * 4 * kPerWord + 2 * kPerWord]);
      unpack_word<T>(u.w, &out[c * 4 * kPerWord + 3 * kPerWord]);
    }
  } else if constexpr (kBytes == 8) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    unpack_word<T>(u.x, &out[0]);
    unpack_word<T>(u.y, &out[kPerWord]);
  } else {
    unpack_word<T>(*reinterpret_cast<const unsigned int*>(p), &out[0]);
  }
}

// cp.async of `kBytes` (4, 8, 16 or 32) from global to shared memory, both
// aligned to min(kBytes, 16)
template <int kBytes>
__device__ __forceinline__ void cp_async_row(void* dst, const void* src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  if constexpr (kBytes <= 16) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(d), "l"(src), "n"(kBytes) : "memory");
  } else {
    static_assert(kBytes == 32, "row bytes per lane");
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d + 16),
                 "l"(static_cast<const char*>(src) + 16)
                 : "memory");
  }
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

constexpr int kStreamWarps = 8;  // warps per CTA of the pipelined compressor

// Prefill compression with the stream kept in flight: each warp walks its
// blocks (grid stride over (b, h, block)) through an NST-stage ring of
// shared-memory copies of the blocks' R token rows, NST - 1 blocks ahead of
// the one it encodes. Lane l copies and later reads only its own VEC channels
// of every row, so its own cp.async completion orders its reads. The
// arithmetic is encode_block, unchanged: codes are bitwise those of the
// unpipelined path and of the append kernel. The first B * H warps also copy
// their (b, h)'s T mod R remaining tokens into the raw tail. SC, RC > 0:
// S and R fixed at compile time (encode_block's compile-time form, the same
// codes).
template <int VEC, typename TIn, typename TOut, int NST, int SC = 0, int RC = 0>
__global__ void __launch_bounds__(kStreamWarps * 32, (SC > 0 && NST == 2) ? 3 : 2)
    compress_stream_kernel(CompressArgs a, BasisF64 basis) {
  extern __shared__ __align__(16) uint8_t csm[];
  constexpr int kLaneBytes = VEC * int(sizeof(TIn));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nw = int64_t(gridDim.x) * kStreamWarps;
  const int64_t w0 = int64_t(blockIdx.x) * kStreamWarps + warp;
  const int64_t stage_bytes = int64_t(a.R) * a.D * int64_t(sizeof(TIn));
  uint8_t* ring = csm + warp * NST * stage_bytes;
  const TIn* x = static_cast<const TIn*>(a.x);

  // walks this warp's items it = w0, w0 + nw, ... as (block n, stream bh)
  // cursors advanced without 64-bit divisions (one up front)
  struct Cursor {
    int64_t n, bh;
  };
  const int64_t step_bh = nw / a.n_full, step_n = nw - step_bh * a.n_full;
  auto advance = [&](Cursor& cur) {
    cur.n += step_n;
    cur.bh += step_bh;
    if (cur.n >= a.n_full) {
      cur.n -= a.n_full;
      ++cur.bh;
    }
  };
  Cursor ci{w0 % a.n_full, w0 / a.n_full};  // next block to issue
  Cursor cc = ci;                           // next block to encode
  const int64_t n_bh = int64_t(a.B) * a.H;
  // (b, h) of a stream index, in 32 bits whenever the index fits
  const bool narrow = n_bh <= int64_t(0xffffffffLL);
  auto split_bh = [&](int64_t bh, int64_t& b, int64_t& h) {
    if (narrow) {
      const uint32_t u = uint32_t(bh), hh = uint32_t(a.H);
      h = u % hh;
      b = u / hh;
    } else {
      h = bh % a.H;
      b = bh / a.H;
    }
  };
  auto issue = [&](int st) {
    if (ci.bh < n_bh) {
      int64_t b, h;
      split_bh(ci.bh, b, h);
      const TIn* src = x + b * a.xs_b + h * a.xs_h + ci.n * a.R * a.xs_t + lane * VEC;
      uint8_t* dst = ring + st * stage_bytes + lane * kLaneBytes;
      for (int t = 0; t < a.R; ++t)
        cp_async_row<kLaneBytes>(dst + int64_t(t) * a.D * int64_t(sizeof(TIn)), src + t * a.xs_t);
    }
    cp_async_commit();  // possibly empty: keeps one group per ring slot
    advance(ci);
  };

#pragma unroll
  for (int s = 0; s < NST - 1; ++s) issue(s);
  for (int64_t k = 0; cc.bh < n_bh; ++k) {
    issue(int((k + NST - 1) % NST));
    cp_async_wait<NST - 1>();
    int64_t b, h;
    split_bh(cc.bh, b, h);
    const int64_t n = cc.n;
    const TIn* rows = reinterpret_cast<const TIn*>(ring + (k % NST) * stage_bytes) + lane * VEC;
    TOut* blk = static_cast<TOut*>(a.out.coeffs) + b * a.out.cs_b + h * a.out.cs_h +
                (a.slot0 + n) * a.S * a.D;
    float* scl = a.out.scales ? a.out.scales + b * a.out.ss_b + h * a.out.ss_h + (a.slot0 + n) * a.S
                              : nullptr;
    encode_block<TOut, VEC, SC, RC>(
        [&](int t, float (&xf)[VEC]) { load_vec_plain<TIn, VEC>(rows + t * a.D, xf); }, a.R, a.S, a.D,
        lane, basis, blk, scl);
    advance(cc);
  }
  cp_async_wait<0>();
  if (a.tail != nullptr && w0 < int64_t(a.B) * a.H) {
    const int h = int(w0 % a.H), b = int(w0 / a.H);
    const TIn* src = x + b * a.xs_b + h * a.xs_h + a.n_full * a.R * a.xs_t + lane * VEC;
    TIn* dst = static_cast<TIn*>(a.tail) + b * a.ts_b + h * a.ts_h + lane * VEC;
    for (int i = 0; i < a.n_rem; ++i) {
      float xv[VEC];
      load_vec<TIn, VEC>(src + i * a.xs_t, xv);
      store_row<TIn, VEC>(dst + int64_t(i) * a.D, xv);
    }
  }
}

struct AppendStream {
  const void* src;  // new token (B, H, 1, D)
  int64_t src_b, src_h;
  void* tail;
  int64_t ts_b, ts_h;
  StreamOut out;
};

struct AppendArgs {
  AppendStream st[2];
  int B, H, R, S, D;
  int len;       // tail rows before this token
  int complete;  // len + 1 == R: archive the block into `slot`
  int64_t slot;
};

template <int VEC, typename TIn, typename TOutK, typename TOutV>
__global__ void __launch_bounds__(256) append_step_kernel(AppendArgs a, BasisF64 basis) {
  // a decode attention launched with FC_DECODE_OVERLAP may start streaming
  // the older archive blocks now: this kernel writes only the tails and the
  // block it completes, which that attention reads after its dependency wait
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // launched as a programmatic dependent: nothing is read or written before
  // the preceding work has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t bh_total = int64_t(a.B) * a.H;
  if (w >= 2 * bh_total) return;
  const int s = int(w / bh_total);
  const int64_t bh = w % bh_total;
  const int h = int(bh % a.H), b = int(bh / a.H);
  const AppendStream& st = a.st[s];
  float xn[VEC];
  load_vec<TIn, VEC>(static_cast<const TIn*>(st.src) + b * st.src_b + h * st.src_h + lane * VEC, xn);
  TIn* trow = static_cast<TIn*>(st.tail) + b * st.ts_b + h * st.ts_h + lane * VEC;
  if (!a.complete) {
    store_row<TIn, VEC>(trow + int64_t(a.len) * a.D, xn);
    return;
  }
  // the block completes: rows 0..R-2 come from the tail, row R-1 is the new token
  auto row_at = [&](int t, float (&xf)[VEC]) {
    if (t < a.R - 1) {
      load_vec<TIn, VEC>(trow + int64_t(t) * a.D, xf);
    } else {
#pragma unroll
      for (int v = 0; v < VEC; ++v) xf[v] = xn[v];
    }
  };
  const StreamOut& o = st.out;
  float* scl = o.scales ? o.scales + b * o.ss_b + h * o.ss_h + a.slot * a.S : nullptr;
  if (s == 0) {
    TOutK* blk = static_cast<TOutK*>(o.coeffs) + b * o.cs_b + h * o.cs_h + a.slot * a.S * a.D;
    encode_block<TOutK, VEC>(row_at, a.R, a.S, a.D, lane, basis, blk, scl);
  } else {
    TOutV* blk = static_cast<TOutV*>(o.coeffs) + b * o.cs_b + h * o.cs_h + a.slot * a.S * a.D;
    encode_block<TOutV, VEC>(row_at, a.R, a.S, a.D, lane, basis, blk, scl);
  }
}

struct CopyArgs {
  const uint8_t* src_c;
  uint8_t* dst_c;
  int64_t src_cb, src_ch, dst_cb, dst_ch;  // byte strides
  int64_t bytes_per_head;                  // multiple of 16
  const float* src_s;
  float* dst_s;
  int64_t src_sb, src_sh, dst_sb, dst_sh;  // element strides
  int64_t scales_per_head;
  int H;
};

__global__ void __launch_bounds__(256) archive_copy_kernel(CopyArgs a) {
  const int bh = blockIdx.y;
  const int h = bh % a.H, b = bh / a.H;
  const uint4* s = reinterpret_cast<const uint4*>(a.src_c + b * a.src_cb + h * a.src_ch);
  uint4* d = reinterpret_cast<uint4*>(a.dst_c + b * a.dst_cb + h * a.dst_ch);
  const int64_t n16 = a.bytes_per_head / 16;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += int64_t(gridDim.x) * blockDim.x)
    d[i] = s[i];
  if (a.src_s) {
    const float* ss = a.src_s + b * a.src_sb + h * a.src_sh;
    float* ds = a.dst_s + b * a.dst_sb + h * a.dst_sh;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < a.scales_per_head;
         i += int64_t(gridDim.x) * blockDim.x)
      ds[i] = ss[i];
  }
}

// ------------------------------------------------------------ dispatch

template <typename F>
int dispatch_vec(int D, F&& f) {
  switch (D) {
    case 32: return f(std::integral_constant<int, 1>{});
    case 64: return f(std::integral_constant<int, 2>{});
    case 128: return f(std::integral_constant<int, 4>{});
    case 256: return f(std::integral_constant<int, 8>{});
    default: return FC_ERR_UNSUPPORTED;
  }
}

template <typename F>
int dispatch_in(int dt, F&& f) {
  if (dt == FC_DTYPE_BF16) return f(__nv_bfloat16{});
  if (dt == FC_DTYPE_F32) return f(float{});
  return FC_ERR_UNSUPPORTED;
}

template <typename F>
int dispatch_out(int dt, F&& f) {
  if (dt == FC_DTYPE_I8) return f(int8_t{});
  if (dt == FC_DTYPE_BF16) return f(__nv_bfloat16{});
  if (dt == FC_DTYPE_F32) return f(float{});
  return FC_ERR_UNSUPPORTED;
}

StreamOut stream_out(const fc_archive* a) {
  StreamOut o;
  o.coeffs = a->coeffs;
  o.scales = a->scales;
  o.cs_b = a->coeff_stride_b;
  o.cs_h = a->coeff_stride_h;
  o.ss_b = a->scale_stride_b;
  o.ss_h = a->scale_stride_h;
  return o;
}

}  // namespace
}  // namespace fc

using namespace fc;

extern "C" int fc_compress_blocks(const void* x, int32_t x_dtype, const int64_t* x_strides,
                                  int64_t T, fc_archive* arc, fc_tail* tail, fc_stream stream) {
  if (!x || !x_strides || T < 0) return FC_ERR_INVALID;
  int st = check_archive(arc);
  if (st != FC_OK) return st;
  if (x_dtype != FC_DTYPE_BF16 && x_dtype != FC_DTYPE_F32) return FC_ERR_INVALID;
  if (x_strides[3] != 1 || x_strides[0] < 0 || x_strides[1] < 0 || x_strides[2] < 0)
    return FC_ERR_INVALID;
  const int esz = dtype_size(x_dtype);
  if (!aligned16(x) || (x_strides[0] * esz) % 16 || (x_strides[1] * esz) % 16 ||
      (x_strides[2] * esz) % 16)
    return FC_ERR_INVALID;
  const int64_t n_full = T / arc->R;
  const int n_rem = int(T - n_full * arc->R);
  if (tail) {
    st = check_tail(tail, arc, n_rem == 0);
    if (st != FC_OK) return st;
    if (tail->len != 0 || tail->dtype != x_dtype) return FC_ERR_INVALID;
  }
  if (arc->n_blocks + n_full > arc->capacity) return FC_ERR_CAPACITY;
  const bool copy_tail = tail && n_rem > 0;
  if (n_full == 0 && !copy_tail) {
    return FC_OK;
  }
  CompressArgs a;
  a.x = x;
  a.xs_b = x_strides[0];
  a.xs_h = x_strides[1];
  a.xs_t = x_strides[2];
  a.B = int(arc->B);
  a.H = int(arc->H);
  a.R = arc->R;
  a.S = arc->S;
  a.D = int(arc->D);
  a.n_full = n_full;
  a.slot0 = arc->n_blocks;
  a.out = stream_out(arc);
  a.tail = copy_tail ? tail->data : nullptr;
  a.ts_b = tail ? tail->stride_b : 0;
  a.ts_h = tail ? tail->stride_h : 0;
  a.n_rem = n_rem;
  BasisF64 basis;
  make_basis_f64(arc->codec, arc->R, arc->S, &basis);
  const int64_t warps = arc->B * arc->H * n_full + (copy_tail ? arc->B * arc->H : 0);
  const int64_t grid = (warps + 7) / 8;
  if (grid > 0x7fffffffLL) return FC_ERR_UNSUPPORTED;
  // the pipelined compressor when a lane's share of a row is a whole word and
  // its ring fits (three stages, two CTAs per SM; else two stages); the
  // direct-load kernel otherwise
  const int64_t stage_bytes = int64_t(arc->R) * arc->D * esz;
  const int lane_bytes = int(arc->D / 32) * esz;
  const int nst = 3 * kStreamWarps * stage_bytes <= 100 * 1024 ? 3
                  : 2 * kStreamWarps * stage_bytes <= 200 * 1024 ? 2 : 0;
  const bool pipelined = nst > 0 && lane_bytes >= 4 && n_full > 0;
  st = dispatch_vec(a.D, [&](auto vec) {
    return dispatch_in(x_dtype, [&](auto tin) {
      return dispatch_out(arc->coeff_dtype, [&](auto tout) {
        using TIn = decltype(tin);
        using TOut = decltype(tout);
        constexpr int VEC = decltype(vec)::value;
        if constexpr (VEC * sizeof(TIn) >= 4) {
          if (pipelined) {
            size_t smem = size_t(kStreamWarps) * nst * stage_bytes;
            const int64_t need = (arc->B * arc->H * n_full + kStreamWarps - 1) / kStreamWarps;
            const int64_t g_tail = (copy_tail ? (arc->B * arc->H + kStreamWarps - 1) / kStreamWarps : 0);
            auto kern = nst == 3 ? compress_stream_kernel<VEC, TIn, TOut, 3> : compress_stream_kernel<VEC, TIn, TOut, 2>;
            // the decode workloads' geometries (D = 128, bf16 tokens, three
            // stages) with S and R fixed at compile time
            int per_sm = nst == 3 ? 2 : 1;
            if constexpr (VEC == 4 && std::is_same<TIn, __nv_bfloat16>::value &&
                          !std::is_same<TOut, float>::value) {
              // two stages, three CTAs per SM (more warps in flight)
              if (nst == 3 && arc->codec == FC_CODEC_DCT) {
                const int nst2 = 2;
                bool fixed = true;
                if (arc->S == 2 && arc->R == 8) kern = compress_stream_kernel<VEC, TIn, TOut, 2, 2, 8>;
                else if (arc->S == 3 && arc->R == 8) kern = compress_stream_kernel<VEC, TIn, TOut, 2, 3, 8>;
                else if (arc->S == 4 && arc->R == 16) kern = compress_stream_kernel<VEC, TIn, TOut, 2, 4, 16>;
                else fixed = false;
                if (fixed) {
                  smem = size_t(kStreamWarps) * nst2 * stage_bytes;
                  per_sm = 3;
                }
              }
            }
            const int64_t cap = int64_t(sm_count()) * per_sm;  // one resident wave
            const int64_t g = need < cap ? need : cap;
            const unsigned grid_p = unsigned(g > g_tail ? g : g_tail);
            if (smem > 48 * 1024 &&
                cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
              return int(FC_ERR_CUDA);
            kern<<<grid_p, kStreamWarps * 32, smem, stream>>>(a, basis);
            return cuda_status(cudaGetLastError());
          }
        }
        compress_blocks_kernel<VEC, TIn, TOut><<<unsigned(grid), 256, 0, stream>>>(a, basis);
        return cuda_status(cudaGetLastError());
      });
    });
  });
  if (st != FC_OK) return st;
  arc->n_blocks += n_full;
  if (copy_tail) tail->len = n_rem;
  return FC_OK;
}

extern "C" int fc_append_step(const void* k_new, const void* v_new, int32_t dtype,
                              const int64_t* k_strides, const int64_t* v_strides, fc_archive* ka,
                              fc_archive* va, fc_tail* kt, fc_tail* vt, fc_stream stream) {
  if (!k_new || !v_new || !k_strides || !v_strides) return FC_ERR_INVALID;
  int st = check_archive(ka);
  if (st != FC_OK) return st;
  st = check_archive(va);
  if (st != FC_OK) return st;
  if (ka->B != va->B || ka->H != va->H || ka->R != va->R || ka->S != va->S || ka->D != va->D ||
      ka->n_blocks != va->n_blocks)
    return FC_ERR_INVALID;
  st = check_tail(kt, ka, false);
  if (st != FC_OK) return st;
  st = check_tail(vt, va, false);
  if (st != FC_OK) return st;
  if (kt->len != vt->len || kt->dtype != dtype || vt->dtype != dtype) return FC_ERR_INVALID;
  if (k_strides[3] != 1 || v_strides[3] != 1) return FC_ERR_INVALID;
  const int esz = dtype_size(dtype);
  if (!aligned16(k_new) || !aligned16(v_new) || (k_strides[0] * esz) % 16 ||
      (k_strides[1] * esz) % 16 || (v_strides[0] * esz) % 16 || (v_strides[1] * esz) % 16)
    return FC_ERR_INVALID;
  const bool complete = kt->len + 1 == ka->R;
  if (complete && (ka->n_blocks >= ka->capacity || va->n_blocks >= va->capacity))
    return FC_ERR_CAPACITY;
  AppendArgs a;
  const fc_archive* arcs[2] = {ka, va};
  const fc_tail* tails[2] = {kt, vt};
  const void* srcs[2] = {k_new, v_new};
  const int64_t* strides[2] = {k_strides, v_strides};
  for (int s = 0; s < 2; ++s) {
    a.st[s].src = srcs[s];
    a.st[s].src_b = strides[s][0];
    a.st[s].src_h = strides[s][1];
    a.st[s].tail = tails[s]->data;
    a.st[s].ts_b = tails[s]->stride_b;
    a.st[s].ts_h = tails[s]->stride_h;
    a.st[s].out = stream_out(arcs[s]);
  }
  a.B = int(ka->B);
  a.H = int(ka->H);
  a.R = ka->R;
  a.S = ka->S;
  a.D = int(ka->D);
  a.len = kt->len;
  a.complete = complete ? 1 : 0;
  a.slot = ka->n_blocks;
  BasisF64 basis;
  make_basis_f64(ka->codec, ka->R, ka->S, &basis);
  const int64_t warps = 2 * ka->B * ka->H;
  const int64_t grid = (warps + 7) / 8;
  st = dispatch_vec(a.D, [&](auto vec) {
    return dispatch_in(dtype, [&](auto tin) {
      return dispatch_out(ka->coeff_dtype, [&](auto tk) {
        return dispatch_out(va->coeff_dtype, [&](auto tv) {
          // a programmatic dependent launch whose first action is the
          // dependency wait: same ordering as a plain launch, but the kernel
          // (and, through its early trigger, a decode attention queued after
          // it with FC_DECODE_OVERLAP) can be scheduled while the preceding
          // kernel drains
          cudaLaunchConfig_t cfg = {};
          cfg.gridDim = dim3(unsigned(grid));
          cfg.blockDim = dim3(256);
          cfg.stream = stream;
          cudaLaunchAttribute attr[1];
          attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
          attr[0].val.programmaticStreamSerializationAllowed = 1;
          cfg.attrs = attr;
          cfg.numAttrs = 1;
          return cuda_status(cudaLaunchKernelEx(
              &cfg, append_step_kernel<decltype(vec)::value, decltype(tin), decltype(tk), decltype(tv)>, a,
              basis));
        });
      });
    });
  });
  if (st != FC_OK) return st;
  if (complete) {
    ka->n_blocks += 1;
    va->n_blocks += 1;
    kt->len = 0;
    vt->len = 0;
  } else {
    kt->len += 1;
    vt->len += 1;
  }
  return FC_OK;
}

extern "C" int fc_archive_copy_prefix(const fc_archive* src, fc_archive* dst, fc_stream stream) {
  int st = check_archive(src);
  if (st != FC_OK) return st;
  st = check_archive(dst);
  if (st != FC_OK) return st;
  if (src->B != dst->B || src->H != dst->H || src->R != dst->R || src->S != dst->S ||
      src->D != dst->D || src->coeff_dtype != dst->coeff_dtype)
    return FC_ERR_INVALID;
  if (dst->capacity < src->n_blocks) return FC_ERR_CAPACITY;
  if (src->n_blocks > 0) {
    const int64_t esz = dtype_size(src->coeff_dtype);
    CopyArgs a;
    a.src_c = static_cast<const uint8_t*>(src->coeffs);
    a.dst_c = static_cast<uint8_t*>(dst->coeffs);
    a.src_cb = src->coeff_stride_b * esz;
    a.src_ch = src->coeff_stride_h * esz;
    a.dst_cb = dst->coeff_stride_b * esz;
    a.dst_ch = dst->coeff_stride_h * esz;
    a.bytes_per_head = src->n_blocks * src->S * src->D * esz;
    a.src_s = src->scales;
    a.dst_s = dst->scales;
    a.src_sb = src->scale_stride_b;
    a.src_sh = src->scale_stride_h;
    a.dst_sb = dst->scale_stride_b;
    a.dst_sh = dst->scale_stride_h;
    a.scales_per_head = src->scales ? src->n_blocks * src->S : 0;
    a.H = int(src->H);
    const int64_t bh = src->B * src->H;
    if (bh > 65535) return FC_ERR_UNSUPPORTED;
    int64_t gx = (a.bytes_per_head / 16 + 255) / 256;
    if (gx > 1024) gx = 1024;
    if (gx < 1) gx = 1;
    archive_copy_kernel<<<dim3(unsigned(gx), unsigned(bh)), 256, 0, stream>>>(a);
    st = cuda_status(cudaGetLastError());
    if (st != FC_OK) return st;
  }
  dst->n_blocks = src->n_blocks;
  return FC_OK;
}
