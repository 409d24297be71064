// Tensor-core decode attention for int8 K and V archives (sm_100a).
//
// Same computation as the portable kernel (flashcodec/triton_attention.py;
// flashcodec-kv README, "Materialization-free decode attention"): per block
// s = C_k q, logits = sigma A s, online softmax, w = p A, acc += w C_v, the
// raw tail folded into the same softmax, split-K partials and a combine.
//
// The two contractions run on the 5th-generation tensor cores straight from
// the int8 archive bytes, so no code is ever converted on the CUDA cores:
//
//   K side  S_int[row][n] = sum_d C_k[row][d] * Lq[n][d]
//           (tcgen05.mma kind::i8, M = 128 coefficient rows, N = 16 or 32,
//           K = D = 128). Lq holds each query head as three 7-bit int8 limbs
//           under one power-of-two exponent per head, which represents the
//           fp32 query to 2^-21 of its largest entry; the int32 sums are exact,
//           so s = scale_k * sum_limbs 2^e * S_int reproduces C_k q to fp32
//           accuracy.
//   V side  Acc_int[d][n] = sum_row C_v[row][d] * Lw[n][row]
//           (kind::i8, M = D = 128 with the V tile read MN-major, K = 128
//           rows). Lw holds w * scale_v as three int8 limbs under one
//           power-of-two exponent per (tile, head), chosen from the bound
//           |w_j| <= p_max(tile) sqrt(R) (the columns of A are unit vectors);
//           the int32 sums are exact.
//
// Warp roles. One TMA thread keeps two rings full: K tiles (128 rows x 128
// codes, 128-byte swizzle), recycled as soon as their K-side MMA completes,
// and V tiles together with the tile's K and V scales, recycled when the
// V-side MMA completes. Two MMA warps issue the K-side MMA of each tile as
// soon as it lands and the V-side MMA as soon as its W is written. NG = 4
// compute groups of four warps (3 when G or S is 8, for registers) take the
// tiles in turn (tile i -> group i mod NG), each with its own online-softmax
// state, so NG tiles are in the softmax at once; the groups' states merge at
// the end of the chunk.
//
// Inside a group, thread t first owns coefficient row t (its TMEM lane) and
// converts the K sums of all heads; a warp-local transpose through shared
// memory then gives each lane whole (block, head) items, so a lane computes
// the R logits of a block from its S scores with the basis as compile-time
// constant operands, takes the R exponentials, and folds them back into the S
// weights w_j without any cross-lane reduction. One named barrier per tile
// exchanges the per-warp maxima. The V epilogue of a tile (thread t = channel
// d, every head) runs one group iteration later, so the V-side MMA overlaps
// the group's next softmax. Integer<->float conversions of the limbs use the
// 1.5 * 2^23 addition (exact for |x| < 2^22), which keeps them on the FMA
// pipes.
//
// Every wait on an mbarrier is bounded; on timeout the kernel records an
// error in the workspace status word, stops issuing work, drains what it
// issued (also bounded), frees its TMEM and returns.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "fc_decode.cuh"
#include "fc_tc_ptx.cuh"

namespace fc {
namespace tc {

constexpr int kRows = 128;  // coefficient rows per tile
constexpr int kD = 128;     // head dim served by this kernel
constexpr uint32_t kTileBytes = kRows * kD;
constexpr uint32_t kScaleBytes = kRows * 4;
constexpr unsigned long long kWaitCycles = 4000000000ull;  // ~2 s at 2 GHz
constexpr unsigned long long kStallCycles = 1ull << 20;     // the test hook's wait
constexpr int kFinBar = 8;   // named barrier over every compute warp
constexpr float kMagic = 12582912.f;  // 1.5 * 2^23
constexpr int kMagicBits = 0x4B400000;

__host__ __device__ constexpr int pad16(int x) { return (x + 15) / 16 * 16; }

template <int G, int S, int TPT>
struct Cfg {
  static constexpr int R = S * TPT;
  static constexpr int TB = kRows / S;             // blocks per tile
  static constexpr int BW = 32 / S;                // blocks per warp
  static constexpr int NI = G >= S ? G / S : 1;    // (block, head) items per lane
  // compute groups of four warps (three where a lane's items need more
  // registers than four groups leave)
  static constexpr int NG = (S == 8 || G == 8) ? 3 : 4;
  static constexpr int HPG = (G + NG - 1) / NG;    // heads per group in the final merge
  static constexpr int NP = pad16(3 * G);          // MMA N: three limb columns per head
  static constexpr int NKS = 4;                    // K ring stages
  static constexpr int NVS = NP == 16 ? 7 : 6;     // V ring stages
  static constexpr int kThreads = 128 * NG + 96;   // + TMA, K-MMA and V-MMA warps
  // per group 2 K and 2 V buffers, allocated as a power of two
  static constexpr uint32_t kTmemCols = 4 * NP * NG <= 256 ? 256 : 512;
  static constexpr uint32_t LBO = 16 * NP;         // W operand: K-direction core-matrix stride
  static constexpr int XP = S * (G + 1);           // transpose scratch floats per block
  static constexpr int XW = BW * XP;               // ... per warp
  // shared memory (offsets from a 1024-byte aligned base)
  static constexpr uint32_t kt = 0;
  static constexpr uint32_t vt = kt + NKS * kTileBytes;
  static constexpr uint32_t qb = vt + NVS * kTileBytes;       // K-major SW128, NP rows x 128 B
  static constexpr uint32_t sc = qb + NP * 128;               // per V stage: K scales, V scales
  static constexpr uint32_t wb = sc + NVS * 2 * kScaleBytes;  // NG x 2 W buffers
  static constexpr uint32_t xs = wb + NG * 2 * NP * 128;     // transpose scratch, 4 NG warps
  static constexpr uint32_t red = xs + NG * 4 * XW * 4;      // NG x 2 x (G + 1) x 4 floats
  static constexpr uint32_t qu = red + NG * 2 * (G + 1) * 16;  // G limb units of q
  static constexpr uint32_t qs = qu + 64;                     // 4 x G floats: |q| maxima
  static constexpr uint32_t bars = qs + 128;
  static constexpr int kBars = 2 * NKS + 2 * NVS + 10 * NG + 1;
  static constexpr uint32_t misc = bars + kBars * 8;          // tmem slot, abort, last
  static constexpr uint32_t bytes = misc + 16;
  static constexpr uint32_t alloc = bytes + 1024;             // alignment slack
  static_assert(alloc <= 232448, "shared memory");
  static_assert((NG * G * (kD + 5) + 4) * 4 <= int(NKS * kTileBytes), "merge scratch");
  static_assert(4 * NP * NG <= 512, "TMEM allocation");
  static_assert(NI * R <= 32, "logits per lane");
  static_assert(R * HPG <= XW, "tail batch scratch");
};

struct TcArgs {
  DecodeArgs d;
  int tiles_per_head;
};

// The problems of one launch (the layers of fc_decode_step_layers, or the
// one problem of a single call): CTA x serves problem p for
// cta_end[p - 1] <= x < cta_end[p]. Passed as a __grid_constant__ parameter,
// so the tensor maps are addressed in parameter space.
template <int NL>
struct TcBatch {
  CUtensorMap maps[NL][4];  // K codes, V codes, K scales, V scales
  TcArgs prob[NL];
  int cta_end[NL];
  int n;
};

// The DCT basis rows the kernel needs, sized for its (S, R): fp32 for the
// attention arithmetic, fp64 for encoding a block in the fused decode step
// (the same values as the codec's). A small parameter block keeps launches
// cheap.
template <int S, int R>
struct TcBasis {
  float m[S][R];
  double m64[S][R];
};

template <int S, int R>
struct Basis64View {  // encode_block indexes basis.m[j][t]
  const double (&m)[S][R];
  static constexpr int32_t mirror = R % 2 == 0 ? 1 : 0;  // the DCT rows
};

__device__ __forceinline__ float pow2i(int e) {
  e = max(-126, min(127, e));
  return __int_as_float((e + 127) << 23);
}

// exponent E with |x| < 2^E for finite x > 0 (-126 for 0 or subnormal x)
__device__ __forceinline__ int exp_above(float x) {
  const int ef = (__float_as_int(x) >> 23) & 0xff;
  return ef == 0 ? -126 : ef - 126;
}

// exact int32 -> float for |v| < 2^22
__device__ __forceinline__ float i2f_small(uint32_t v) {
  return __fsub_rn(__int_as_float(int(v) + kMagicBits), kMagic);
}

// x ~ L0 + L1 / 128 + L2 / 16384 for x in (-64, 64), limbs rounded to nearest
// even; returns each limb in the low byte of a word
__device__ __forceinline__ void limb_bytes(float x, uint32_t& b0, uint32_t& b1, uint32_t& b2) {
  const float t0 = __fadd_rn(x, kMagic);
  const float y1 = __fmul_rn(__fsub_rn(x, __fsub_rn(t0, kMagic)), 128.f);
  const float t1 = __fadd_rn(y1, kMagic);
  const float y2 = __fmul_rn(__fsub_rn(y1, __fsub_rn(t1, kMagic)), 128.f);
  const float t2 = __fadd_rn(y2, kMagic);
  b0 = __float_as_uint(t0);
  b1 = __float_as_uint(t1);
  b2 = __float_as_uint(t2);
}

__device__ __forceinline__ float unlimb3(uint32_t c0, uint32_t c1, uint32_t c2) {
  return fmaf(i2f_small(c2), 1.f / 16384.f, fmaf(i2f_small(c1), 1.f / 128.f, i2f_small(c0)));
}

// byte offset of element (row n, column k) in a 128-byte-swizzled K-major
// operand whose rows are 128 bytes (1024-byte-aligned atoms of 8 rows)
__device__ __forceinline__ uint32_t sw128_offset(int n, int k) {
  return uint32_t(n) * 128u + ((uint32_t(k >> 4) ^ uint32_t(n & 7)) << 4) + uint32_t(k & 15);
}

// byte offset of W[n][k] (column n = head limb, k = tile row) in the K-major
// operand without swizzle: 8 x 16-byte core matrices, N-adjacent ones 128 B
// apart, K-adjacent ones LBO apart
template <uint32_t LBO>
__device__ __forceinline__ uint32_t w_offset(int n, int k) {
  return uint32_t(k >> 4) * LBO + uint32_t(n >> 3) * 128u + uint32_t(n & 7) * 16u + uint32_t(k & 15);
}

// stores the low bytes of S words as S consecutive bytes
template <int S>
__device__ __forceinline__ void store_bytes(uint8_t* p, const uint32_t (&v)[S]) {
  if constexpr (S == 1) {
    *p = uint8_t(v[0]);
  } else if constexpr (S == 2) {
    *reinterpret_cast<uint16_t*>(p) = uint16_t(__byte_perm(v[0], v[1], 0x0040));
  } else if constexpr (S == 4) {
    *reinterpret_cast<uint32_t*>(p) =
        __byte_perm(__byte_perm(v[0], v[1], 0x0040), __byte_perm(v[2], v[3], 0x0040), 0x5410);
  } else {
    static_assert(S == 8, "S");
    const uint32_t lo =
        __byte_perm(__byte_perm(v[0], v[1], 0x0040), __byte_perm(v[2], v[3], 0x0040), 0x5410);
    const uint32_t hi =
        __byte_perm(__byte_perm(v[4], v[5], 0x0040), __byte_perm(v[6], v[7], 0x0040), 0x5410);
    *reinterpret_cast<uint2*>(p) = make_uint2(lo, hi);
  }
}

template <int N>
__device__ __forceinline__ void load_floats(const float* p, float (&v)[N]) {
  if constexpr (N == 1) {
    v[0] = p[0];
  } else if constexpr (N == 2) {
    const float2 x = *reinterpret_cast<const float2*>(p);
    v[0] = x.x;
    v[1] = x.y;
  } else {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      const float4 x = *reinterpret_cast<const float4*>(p + i);
      v[i] = x.x;
      v[i + 1] = x.y;
      v[i + 2] = x.z;
      v[i + 3] = x.w;
    }
  }
}

template <int N>
__device__ __forceinline__ float pick(const float (&v)[N], int i) {
  float r = v[0];
#pragma unroll
  for (int k = 1; k < N; ++k) r = (k == i) ? v[k] : r;
  return r;
}

// The aligned 32-bit word that holds element `idx` of a bf16 or fp32 tensor
// whose base and row strides are multiples of 16 bytes (the raw tails and a
// fused step's new tokens; bf16: the pair the element belongs to), and the
// element's value from that word given its column `col` in the row (the
// parity of col and idx agree there).
__device__ __forceinline__ const uint32_t* elem_word(const void* p, int64_t idx, bool f32) {
  const char* c = static_cast<const char*>(p);
  return reinterpret_cast<const uint32_t*>(f32 ? c + idx * 4 : c + (idx & ~int64_t(1)) * 2);
}
__device__ __forceinline__ float word_elem(uint32_t w, int col, bool f32) {
  return __uint_as_float(f32 ? w : ((col & 1) ? (w & 0xffff0000u) : (w << 16)));
}

struct Waiter {
  int* abort;
  uint32_t* status;
  unsigned long long limit;  // clock cycles
  __device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity) {
    if (*reinterpret_cast<volatile int*>(abort)) return false;
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = clock64();
    while (!ptx::mbar_try_wait(bar, parity)) {
      if (*reinterpret_cast<volatile int*>(abort)) return false;
      if (clock64() - t0 > limit) {
        *reinterpret_cast<volatile int*>(abort) = 1;
        if (status) atomicOr(status, 1u);
        return false;
      }
    }
    return true;
  }
};

// bounded wait that ignores the abort flag (draining after an abort)
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = clock64();
  while (!ptx::mbar_try_wait(bar, parity) && clock64() - t0 < kWaitCycles) {
  }
}

// Sums N values per thread over the 128 threads of one warp group (named
// barrier `bar_id`; scratch: 4 warps x 32 floats).
template <int N>
__device__ __forceinline__ void group_sum(float (&v)[N], float* red, int wq, int lane, int bar_id) {
#pragma unroll
  for (int g = 0; g < N; ++g) v[g] = warp_sum(v[g]);
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < N; ++g) red[wq * 32 + g] = v[g];
  }
  ptx::named_bar_sync(bar_id, 128);
#pragma unroll
  for (int g = 0; g < N; ++g) v[g] = red[0 * 32 + g] + red[1 * 32 + g] + red[2 * 32 + g] + red[3 * 32 + g];
  ptx::named_bar_sync(bar_id, 128);
}

// dst[di] = src[si] for a runtime dtype (FC_DTYPE_F32 or FC_DTYPE_BF16), bits copied
__device__ __forceinline__ void copy_elem(const void* dst, int64_t di, const void* src, int64_t si, int dtype) {
  if (dtype == FC_DTYPE_F32)
    const_cast<float*>(static_cast<const float*>(dst))[di] = static_cast<const float*>(src)[si];
  else
    const_cast<unsigned short*>(static_cast<const unsigned short*>(dst))[di] =
        static_cast<const unsigned short*>(src)[si];
}

// Fused decode step: the block completed by the new token (rows 0..R-2 from
// the tail, row R-1 the token) encoded by one warp into archive slot new_slot
// of K (which = 0) or V (which = 1), exactly as the append kernel does.
template <int S, int R>
__device__ __forceinline__ void encode_new_block(const DecodeArgs& a, int which, int lane,
                                                 const TcBasis<S, R>& basis, int b, int h) {
  const Basis64View<S, R> basis64{basis.m64};
  constexpr int VEC = kD / 32;
  const StreamOut& o = which ? a.vout : a.kout;
  const void* tail = which ? a.vt : a.kt;
  const int64_t tb = which ? a.vts_b : a.kts_b, th = which ? a.vts_h : a.kts_h;
  const void* nw = which ? a.vn : a.kn;
  const int64_t nb_ = which ? a.vns_b : a.kns_b, nh = which ? a.vns_h : a.kns_h;
  int8_t* blk = static_cast<int8_t*>(o.coeffs) + b * o.cs_b + h * o.cs_h + a.new_slot * a.S * kD;
  float* scl = o.scales + b * o.ss_b + h * o.ss_h + a.new_slot * a.S;
  auto run = [&](auto tag) {
    using T = decltype(tag);
    const T* trow = static_cast<const T*>(tail) + b * tb + h * th + lane * VEC;
    float xn[VEC];
    load_vec<T, VEC>(static_cast<const T*>(nw) + b * nb_ + h * nh + lane * VEC, xn);
    auto row_at = [&](int t, float (&xf)[VEC]) {
      if (t < R - 1) {
        load_vec<T, VEC>(trow + int64_t(t) * kD, xf);
      } else {
#pragma unroll
        for (int v = 0; v < VEC; ++v) xf[v] = xn[v];
      }
    };
    encode_block<int8_t, VEC>(row_at, R, a.S, kD, lane, basis64, blk, scl);
  };
  if (a.t_dtype == FC_DTYPE_F32)
    run(float(0));
  else
    run(__nv_bfloat16());
}

template <int NP>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NP]) {
  if constexpr (NP == 16) {
    ptx::tmem_ld16(taddr, r);
  } else {
    static_assert(NP == 32, "NP");
    ptx::tmem_ld32(taddr, r);
  }
}

template <int G, int S, int TPT, int NL>
__global__ void __launch_bounds__(Cfg<G, S, TPT>::kThreads, 1)
    decode_tc_kernel(const __grid_constant__ TcBatch<NL> batch, const TcBasis<S, S * TPT> basis) {
  // this CTA's problem
  int prob = 0;
  if constexpr (NL > 1) {
    while (prob + 1 < batch.n && int(blockIdx.x) >= batch.cta_end[prob]) ++prob;
  }
  const int bx_local = int(blockIdx.x) - (prob > 0 ? batch.cta_end[prob - 1] : 0);
  const TcArgs& ta = batch.prob[prob];
  const CUtensorMap& tm_k = batch.maps[prob][0];
  const CUtensorMap& tm_v = batch.maps[prob][1];
  const CUtensorMap& tm_ks = batch.maps[prob][2];
  const CUtensorMap& tm_vs = batch.maps[prob][3];
  using C = Cfg<G, S, TPT>;
  constexpr int R = C::R, NP = C::NP, NI = C::NI, NKS = C::NKS, NVS = C::NVS, XP = C::XP;
  constexpr int NG = C::NG;
  constexpr int NCW = 4 * NG;  // compute warps
  constexpr uint32_t kIdescK = ptx::idesc_i8(128, NP, false, false);
  constexpr uint32_t kIdescV = ptx::idesc_i8(128, NP, true, false);
  constexpr uint32_t kWBytes = NP * 128;  // one W buffer

  const DecodeArgs& a = ta.d;
  extern __shared__ uint8_t smem_raw[];
  // 128-byte swizzle atoms need 1024-byte alignment in the shared window
  uint8_t* sm = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::bars);
  uint64_t* kfull = bars;         // K tile landed (TMA -> K-MMA)
  uint64_t* kfree = kfull + NKS;  // K-side MMA done with the stage (-> TMA)
  uint64_t* vfull = kfree + NKS;  // V tile and both scale rows landed (TMA -> compute, V-MMA)
  uint64_t* vfree = vfull + NVS;  // V-side MMA done with the stage (-> TMA)
  uint64_t* gbar = vfree + NVS;   // per group: kres[2] kemp[2] wrdy[2] vres[2] vemp[2]
  uint64_t* qready = gbar + 10 * NG;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::misc);
  int* abort_flag = reinterpret_cast<int*>(sm + C::misc + 4);
  int* last_flag = reinterpret_cast<int*>(sm + C::misc + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // CTA -> (kv head unit, chunk c of its ns_u): the first bal_rem units take
  // bal_q + 1 chunks, the others bal_q; a unit's tiles split evenly
  int unit, c, ns_u;
  {
    const int bx = bx_local, hi = a.bal_q + 1;
    if (bx < a.bal_rem * hi) {
      unit = bx / hi;
      c = bx - unit * hi;
      ns_u = hi;
    } else {
      const int r = bx - a.bal_rem * hi;
      unit = a.bal_rem + r / a.bal_q;
      c = r - (unit - a.bal_rem) * a.bal_q;
      ns_u = a.bal_q;
    }
  }
  const int h = unit % a.Hk, b = unit / a.Hk;
  const int Hq = a.Hk * G;
  Waiter waiter{abort_flag, a.status, kWaitCycles};

  // chunks of ceil(tiles / ns_u) tiles: the last chunk, which also folds
  // in the raw tail, gets what is left (at most as many tiles as the others)
  const int chunk_tiles = (ta.tiles_per_head + ns_u - 1) / ns_u;
  const int tile0 = c * chunk_tiles;
  const int tile1 = min(tile0 + chunk_tiles, ta.tiles_per_head);
  const int ntiles = max(0, tile1 - tile0);
  const bool producer = warp >= NCW;
  const bool tma_warp = warp == NCW;
  const bool kmma_warp = warp == NCW + 1;  // also owns the TMEM allocation
  const bool vmma_warp = warp == NCW + 2;

  const int grp = producer ? 0 : warp >> 2;  // compute group
  const int w = warp & 3;                    // warp in the group = TMEM lane quadrant
  const int t = tid & 127;                   // thread in the group
  // group 0 reads the query (thread t = channel d). Without FC_DECODE_OVERLAP
  // (or with FC_DECODE_Q_FINAL) it does so before anything else, so that these
  // loads do not queue behind the ring fill; otherwise after the setup barrier
  // and the dependency wait (q comes from the preceding work), while the fill
  // has long been running.
  float qd[G];
  auto load_q = [&]() {
#pragma unroll
    for (int g = 0; g < G; ++g)
      qd[g] = load_any(a.q, b * a.qs_b + (h * G + g) * a.qs_h + t, a.q_dtype) * a.qscale;
  };
  const bool q_after_wait = a.overlap && !a.q_final;
  if (!producer && grp == 0 && !q_after_wait) load_q();

  // TMA thread: issues a K load into stage nk % NKS / a V load (codes and both
  // scale rows) into stage nv % NVS
  // (under FC_DECODE_OVERLAP the head's last tile, which holds the block the
  // preceding work may have just written, waits for that work)
  auto load_k = [&](int nk) {
    if (a.overlap && tile0 + nk == ta.tiles_per_head - 1) ptx::grid_dep_wait();
    const int s = nk % NKS;
    ptx::mbar_arrive_expect_tx(&kfull[s], kTileBytes);
    ptx::tma_load_4d(sm + C::kt + s * kTileBytes, &tm_k, &kfull[s], 0, (tile0 + nk) * kRows, h, b);
  };
  auto load_v = [&](int nv) {
    if (a.overlap && tile0 + nv == ta.tiles_per_head - 1) ptx::grid_dep_wait();
    const int s = nv % NVS;
    const int row0 = (tile0 + nv) * kRows;
    uint8_t* scs = sm + C::sc + s * 2 * kScaleBytes;
    ptx::mbar_arrive_expect_tx(&vfull[s], kTileBytes + 2 * kScaleBytes);
    ptx::tma_load_4d(sm + C::vt + s * kTileBytes, &tm_v, &vfull[s], 0, row0, h, b);
    ptx::tma_load_3d(scs, &tm_ks, &vfull[s], row0, h, b);
    ptx::tma_load_3d(scs + kScaleBytes, &tm_vs, &vfull[s], row0, h, b);
  };
  int nk = 0, nv = 0;  // loads issued (TMA thread)
  if (tma_warp && lane == 0) {
    for (int i = 0; i < NKS; ++i) {
      ptx::mbar_init(&kfull[i], 1);
      ptx::mbar_init(&kfree[i], 1);
    }
    for (int i = 0; i < NVS; ++i) {
      ptx::mbar_init(&vfull[i], 1);
      ptx::mbar_init(&vfree[i], 1);
    }
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tm_k);
    ptx::prefetch_tmap(&tm_v);
    ptx::prefetch_tmap(&tm_ks);
    ptx::prefetch_tmap(&tm_vs);
  }
  if (tid == 0) {
    for (int g = 0; g < NG; ++g)
      for (int x = 0; x < 2; ++x) {
        ptx::mbar_init(&gbar[10 * g + 0 + x], 1);    // kres: K-side MMA committed
        ptx::mbar_init(&gbar[10 * g + 2 + x], 128);  // kemp: the group read the K sums
        ptx::mbar_init(&gbar[10 * g + 4 + x], 128);  // wrdy: the group wrote W
        ptx::mbar_init(&gbar[10 * g + 6 + x], 1);    // vres: V-side MMA committed
        ptx::mbar_init(&gbar[10 * g + 8 + x], 128);  // vemp: the group read the V sums
      }
    ptx::mbar_init(qready, 128);
    *abort_flag = 0;
    *last_flag = 0;
    ptx::fence_mbar_init();
  }
  if (kmma_warp) {
    ptx::tmem_alloc(tmem_slot, C::kTmemCols);
    ptx::tmem_relinquish();
  }

  // barriers and the TMEM address are visible to every warp from here on
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // a dependent launch may be scheduled as SMs free up: it only streams the
  // archive until this grid has completed
  if (a.overlap) ptx::grid_dep_launch();
  if (tma_warp && lane == 0) {
    // fill every stage at once, K and V of a tile together, while group 0
    // prepares the query limbs
    const int fk = min(NKS, ntiles), fv = min(NVS, ntiles);
    for (int i = 0; i < fk || i < fv; ++i) {
      if (i < fk) load_k(i);
      if (i < fv) load_v(i);
    }
    nk = fk;
    nv = fv;
  }

  uint64_t* kres = gbar + 10 * grp;
  uint64_t* kemp = kres + 2;
  uint64_t* wrdy = kres + 4;
  uint64_t* vres = kres + 6;
  uint64_t* vemp = kres + 8;
  const uint32_t tm_grp = tmem + uint32_t(grp * 4 * NP);  // K buffers, then V buffers

  // ---- group 0: the query as three int8 limbs per head (thread t = channel d)
  if (!producer && grp == 0) {
    if (q_after_wait) {
      ptx::grid_dep_wait();
      load_q();
    }
    float* qmx = reinterpret_cast<float*>(sm + C::qs);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mx = warp_max(fabsf(qd[g]));
      if (lane == 0) qmx[w * G + g] = mx;
    }
    ptx::named_bar_sync(1, 128);
    uint8_t* qb = sm + C::qb;
    float* qu = reinterpret_cast<float*>(sm + C::qu);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mx = fmaxf(fmaxf(qmx[g], qmx[G + g]), fmaxf(qmx[2 * G + g], qmx[3 * G + g]));
      const int e = exp_above(mx);
      if (t == 0) qu[g] = pow2i(e - 6);
      uint32_t l0, l1, l2;
      limb_bytes(qd[g] * pow2i(6 - e), l0, l1, l2);
      qb[sw128_offset(3 * g + 0, t)] = uint8_t(l0);
      qb[sw128_offset(3 * g + 1, t)] = uint8_t(l1);
      qb[sw128_offset(3 * g + 2, t)] = uint8_t(l2);
    }
    for (int n = 3 * G; n < NP; ++n) qb[sw128_offset(n, t)] = 0;
    ptx::fence_proxy_async_smem();
    ptx::mbar_arrive(qready);
  }

  if (tma_warp && lane == 0) {
    // ================= TMA thread: both rings, in tile order each, whichever
    // has a free stage (every stage was filled once before the setup barrier)
    unsigned long long t_last = clock64();
    while (nk < ntiles || nv < ntiles) {
      bool prog = false;
      if (nk < ntiles && ptx::mbar_test_wait(&kfree[nk % NKS], uint32_t(nk / NKS - 1) & 1u)) {
        load_k(nk++);
        prog = true;
      }
      if (nv < ntiles && ptx::mbar_test_wait(&vfree[nv % NVS], uint32_t(nv / NVS - 1) & 1u)) {
        load_v(nv++);
        prog = true;
      }
      if (prog) {
        t_last = clock64();
        continue;
      }
      if (*reinterpret_cast<volatile int*>(abort_flag)) break;
      if (clock64() - t_last > kWaitCycles) {
        *reinterpret_cast<volatile int*>(abort_flag) = 1;
        if (a.status) atomicOr(a.status, 1u);
        break;
      }
      __nanosleep(32);
    }
  }
  int mk = 0, mv = 0;  // tiles whose K-side / V-side MMAs were issued
  if (kmma_warp && lane == 0) {
    // ================= K-MMA thread: S_int of each tile into its group's
    // TMEM buffer as soon as it lands
    waiter.wait(qready, 0u);
    if (a.test_stall) {
      // test hook: the next phase of qready, which nothing completes
      Waiter stall{abort_flag, a.status, kStallCycles};
      stall.wait(qready, 1u);
    }
    int i = 0;
    for (; i < ntiles; ++i) {
      const int s = i % NKS, g = i % NG, k = i / NG, x = k & 1;
      uint64_t* gq = gbar + 10 * g;
      if (!waiter.wait(&kfull[s], uint32_t(i / NKS) & 1u)) break;
      if (!waiter.wait(&gq[2 + x], (uint32_t(k >> 1) & 1u) ^ 1u)) break;
      ptx::tc_fence_after();
      const uint32_t ka = ptx::smem_u32(sm + C::kt + s * kTileBytes);
      const uint32_t qa = ptx::smem_u32(sm + C::qb);
      const uint32_t d = tmem + uint32_t(g * 4 * NP + x * NP);
#pragma unroll
      for (int kk = 0; kk < kD / 32; ++kk)
        ptx::mma_i8(d, ptx::desc_sw128(ka + 32 * kk, 16, 1024), ptx::desc_sw128(qa + 32 * kk, 16, 1024),
                    kIdescK, kk > 0 ? 1u : 0u);
      ptx::mma_commit(&kfree[s]);
      ptx::mma_commit(&gq[x]);
    }
    mk = i;
  }
  if (vmma_warp && lane == 0) {
    // ================= V-MMA thread: Acc_int of each tile as soon as its W is
    // written
    int i = 0;
    for (; i < ntiles; ++i) {
      const int s = i % NVS, g = i % NG, k = i / NG, x = k & 1;
      uint64_t* gq = gbar + 10 * g;
      if (!waiter.wait(&vfull[s], uint32_t(i / NVS) & 1u)) break;
      if (!waiter.wait(&gq[4 + x], uint32_t(k >> 1) & 1u)) break;
      if (!waiter.wait(&gq[8 + x], (uint32_t(k >> 1) & 1u) ^ 1u)) break;
      ptx::tc_fence_after();
      const uint32_t va = ptx::smem_u32(sm + C::vt + s * kTileBytes);
      const uint32_t wa = ptx::smem_u32(sm + C::wb + (g * 2 + x) * kWBytes);
      const uint32_t d = tmem + uint32_t(g * 4 * NP + 2 * NP + x * NP);
#pragma unroll
      for (int kk = 0; kk < kRows / 32; ++kk)
        ptx::mma_i8(d, ptx::desc_sw128(va + 4096 * kk, kTileBytes, 1024),
                    ptx::desc_noswizzle(wa + kk * 2 * C::LBO, C::LBO, 128), kIdescV, kk > 0 ? 1u : 0u);
      ptx::mma_commit(&vfree[s]);
      ptx::mma_commit(&gq[6 + x]);
    }
    mv = i;
  }

  // ================= compute groups
  float m_run[G], acc[G];
  float lsum[NI];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY;
    acc[g] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < NI; ++i) lsum[i] = 0.f;
  const int bl = lane / S, jj = lane % S;  // block in the warp, row of the block
  const bool own = G >= S || jj < G;       // lane owns (block, head) items
  if (!producer) {
    // zero this group's W buffers once: the pad columns are never written
    {
      uint4* wz = reinterpret_cast<uint4*>(sm + C::wb + grp * 2 * kWBytes);
      for (int x = t; x < int(2 * kWBytes / 16); x += 128) wz[x] = make_uint4(0u, 0u, 0u, 0u);
    }
    waiter.wait(qready, 0u);
    float qunit[G];  // weight of limb 0 of each head
#pragma unroll
    for (int g = 0; g < G; ++g) qunit[g] = reinterpret_cast<const float*>(sm + C::qu)[g];
    const int bt = w * C::BW + bl;  // block in the tile
    float* xw = reinterpret_cast<float*>(sm + C::xs) + (grp * 4 + w) * C::XW + bl * XP;
    float* rdbase = reinterpret_cast<float*>(sm + C::red) + grp * 2 * (G + 1) * 4;
    uint8_t* wbase = sm + C::wb + grp * 2 * kWBytes;
    const float sqrtR = sqrtf(float(R));
    const uint32_t lane_off = uint32_t(w * 32) << 16;
    float alpha_p[G], wunit_p[G];  // of the tile whose V epilogue is pending
#pragma unroll
    for (int g = 0; g < G; ++g) {
      alpha_p[g] = 1.f;
      wunit_p[g] = 0.f;
    }

    // V epilogue of group iteration kk: acc = alpha acc + W-limb sums
    auto v_epilogue = [&](int kk, const float (&al)[G], const float (&wu)[G]) {
      const int x = kk & 1;
      waiter.wait(&vres[x], uint32_t(kk >> 1) & 1u);
      ptx::tc_fence_after();
      uint32_t vr[NP];
      tmem_ld_cols<NP>(tm_grp + 2 * NP + x * NP + lane_off, vr);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&vemp[x]);
#pragma unroll
      for (int g = 0; g < G; ++g)
        acc[g] = fmaf(acc[g], al[g], wu[g] * unlimb3(vr[3 * g], vr[3 * g + 1], vr[3 * g + 2]));
    };

    int k = 0;
    for (; grp + k * NG < ntiles; ++k) {
      const int i = grp + k * NG;  // tile of the chunk
      const int x = k & 1;
      const int sv = i % NVS;
      const int64_t tile = tile0 + i;
      // the groups start one after another (group g once group g - 1 has
      // written its first W), so the first stages are released early and the
      // rings refill while the other groups work
      if (k == 0 && grp > 0) waiter.wait(&gbar[10 * (grp - 1) + 4], 0u);
      // ---- K sums of my row, every head
      waiter.wait(&kres[x], uint32_t(k >> 1) & 1u);
      ptx::tc_fence_after();
      uint32_t cr[NP];
      tmem_ld_cols<NP>(tm_grp + x * NP + lane_off, cr);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&kemp[x]);
      waiter.wait(&vfull[sv], uint32_t(i / NVS) & 1u);
      const float* scs = reinterpret_cast<const float*>(sm + C::sc + sv * 2 * kScaleBytes);
      const float sk = scs[t];
      // s = scale_k C_k q of my row for every head, transposed through shared
      // memory to (block, head) items: the S scores of each of my blocks' heads
#pragma unroll
      for (int g = 0; g < G; ++g)
        xw[g * S + jj] = (sk * qunit[g]) * unlimb3(cr[3 * g], cr[3 * g + 1], cr[3 * g + 2]);
      __syncwarp();
      float sb[NI][S];
#pragma unroll
      for (int ii = 0; ii < NI; ++ii) load_floats<S>(xw + (own ? jj * NI + ii : 0) * S, sb[ii]);
      float vsc[S];  // V scales of my block
      load_floats<S>(scs + kRows + bt * S, vsc);

      // logits of my items (basis entries are compile-time constant operands).
      // The DCT rows are symmetric, A[R-1-t][j] = (-1)^j A[t][j], so the even-
      // and odd-frequency parts of rows t < R/2 give both halves:
      // logit_t = E_t + O_t, logit_{R-1-t} = E_t - O_t
      const bool live = tile * C::TB + bt < a.nb;
      float lg[NI][R];
      float mx[NI];
#pragma unroll
      for (int ii = 0; ii < NI; ++ii) {
        float m = -INFINITY;
#pragma unroll
        for (int tk = 0; tk < R / 2; ++tk) {
          float ev = basis.m[0][tk] * sb[ii][0];
#pragma unroll
          for (int q = 2; q < S; q += 2) ev = fmaf(basis.m[q][tk], sb[ii][q], ev);
          float od = 0.f;
          if constexpr (S > 1) {
            od = basis.m[1][tk] * sb[ii][1];
#pragma unroll
            for (int q = 3; q < S; q += 2) od = fmaf(basis.m[q][tk], sb[ii][q], od);
          }
          lg[ii][tk] = ev + od;
          lg[ii][R - 1 - tk] = ev - od;
          m = fmaxf(m, fmaxf(lg[ii][tk], lg[ii][R - 1 - tk]));
        }
        m = live && own ? m : -INFINITY;
#pragma unroll
        for (int o = S; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        mx[ii] = m;
      }
      // the tile's largest V scale (scales are >= 0, so their bit patterns
      // order like their values)
      float vm = vsc[0];
#pragma unroll
      for (int q = 1; q < S; ++q) vm = fmaxf(vm, vsc[q]);
      vm = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(vm)));
      // per-warp maxima -> tile maxima (one barrier; slots alternate by tile)
      float* rd = rdbase + x * (G + 1) * 4;
      if (bl == 0 && own) {
#pragma unroll
        for (int ii = 0; ii < NI; ++ii) rd[(jj * NI + ii) * 4 + w] = mx[ii];
      }
      if (lane == 0) rd[G * 4 + w] = vm;
      ptx::named_bar_sync(1 + grp, 128);
      float m_new[G], alpha[G], wunit[G], winv[G];
      {
        const float4 v4 = reinterpret_cast<const float4*>(rd)[G];
        const float vmax = fmaxf(fmaxf(v4.x, v4.y), fmaxf(v4.z, v4.w));
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float4 r4 = reinterpret_cast<const float4*>(rd)[g];
          const float tmax = fmaxf(fmaxf(r4.x, r4.y), fmaxf(r4.z, r4.w));
          m_new[g] = fmaxf(m_run[g], tmax);
          alpha[g] = ptx::ex2(m_run[g] - m_new[g]);
          const int e = exp_above(ptx::ex2(tmax - m_new[g]) * sqrtR * vmax);
          wunit[g] = pow2i(e - 6);
          winv[g] = pow2i(6 - e);
        }
      }
      // p, softmax sums, w_j = sum_t p_t A[t][j], and W = w * scale_v as
      // three int8 limbs: S bytes (my block's rows) of each limb column
      uint8_t* wbuf = wbase + x * kWBytes;
#pragma unroll
      for (int ii = 0; ii < NI; ++ii) {
        if (!own) continue;
        const int hh = jj * NI + ii;
        const float me = live ? pick(m_new, hh) : INFINITY;  // dead blocks: p = 0
        float p[R];
        float ps = 0.f;
#pragma unroll
        for (int tk = 0; tk < R; ++tk) {
          p[tk] = ptx::ex2(lg[ii][tk] - me);
          ps += p[tk];
        }
        lsum[ii] = fmaf(lsum[ii], pick(alpha, hh), ps);
        const float wi = pick(winv, hh);
        // w_j = sum_t p_t A[t][j] over the symmetric halves: with
        // u_t = p_t + p_{R-1-t} (even j) or p_t - p_{R-1-t} (odd j), t < R/2
        float pa[R / 2], pd[R / 2];
#pragma unroll
        for (int tk = 0; tk < R / 2; ++tk) {
          pa[tk] = p[tk] + p[R - 1 - tk];
          pd[tk] = p[tk] - p[R - 1 - tk];
        }
        uint32_t by[3][S];
#pragma unroll
        for (int q = 0; q < S; ++q) {
          float wq = ((q & 1) ? pd[0] : pa[0]) * basis.m[q][0];
#pragma unroll
          for (int tk = 1; tk < R / 2; ++tk) wq = fmaf((q & 1) ? pd[tk] : pa[tk], basis.m[q][tk], wq);
          limb_bytes(wq * vsc[q] * wi, by[0][q], by[1][q], by[2][q]);
        }
#pragma unroll
        for (int l = 0; l < 3; ++l) store_bytes<S>(wbuf + w_offset<C::LBO>(3 * hh + l, bt * S), by[l]);
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(&wrdy[x]);
#pragma unroll
      for (int g = 0; g < G; ++g) m_run[g] = m_new[g];

      // ---- V epilogue of my previous tile (its MMA overlapped this softmax)
      if (k >= 1) v_epilogue(k - 1, alpha_p, wunit_p);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        alpha_p[g] = alpha[g];
        wunit_p[g] = wunit[g];
      }
    }
    if (k >= 1) v_epilogue(k - 1, alpha_p, wunit_p);
  }

  // ---- merge the four groups' states, fold the raw tail, write the partials
  const bool direct = a.fuse && ns_u == 1;
  if (!producer) {
    // softmax sums of my items over the warp's blocks
#pragma unroll
    for (int ii = 0; ii < NI; ++ii)
#pragma unroll
      for (int o = S; o < 32; o <<= 1) lsum[ii] += __shfl_xor_sync(0xffffffffu, lsum[ii], o);
    // the tails, the workspace and out: after the preceding work
    if (a.overlap) ptx::grid_dep_wait();
    // every group is done with both rings: the K ring becomes merge scratch
    ptx::named_bar_sync(kFinBar, 128 * NG);
    float* fm = reinterpret_cast<float*>(sm + C::kt);  // [group][head] running max
    float* fl = fm + (NG * G + 3) / 4 * 4;              // [group][head][warp] sums (16-B aligned)
    float* fa = fl + NG * G * 4;                        // [group][head][channel] acc
    if (t == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) fm[grp * G + g] = m_run[g];
    }
    if (bl == 0 && own) {
#pragma unroll
      for (int ii = 0; ii < NI; ++ii) fl[(grp * G + jj * NI + ii) * 4 + w] = lsum[ii];
    }
#pragma unroll
    for (int g = 0; g < G; ++g) fa[(grp * G + g) * kD + t] = acc[g];
    ptx::named_bar_sync(kFinBar, 128 * NG);

    // group grp finishes heads grp, grp + 4, ...: thread t = channel d
    constexpr int HPG = C::HPG;
    float Mh[HPG], Lh[HPG], Ah[HPG];
#pragma unroll
    for (int y = 0; y < HPG; ++y) {
      const int g = min(grp + NG * y, G - 1);
      float M = -INFINITY;
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        const float4 l4 = reinterpret_cast<const float4*>(fl)[gg * G + g];
        if (l4.x + l4.y + l4.z + l4.w > 0.f) M = fmaxf(M, fm[gg * G + g]);
      }
      float Ls = 0.f, As = 0.f;
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        const float4 l4 = reinterpret_cast<const float4*>(fl)[gg * G + g];
        const float lt = l4.x + l4.y + l4.z + l4.w;
        if (lt > 0.f) {
          const float e = ptx::ex2(fm[gg * G + g] - M);
          Ls = fmaf(lt, e, Ls);
          As = fmaf(fa[(gg * G + g) * kD + t], e, As);
        }
      }
      Mh[y] = M;
      Lh[y] = Ls;
      Ah[y] = As;
    }
    const bool active = grp < G;  // uniform per group
    const bool last_chunk = c == ns_u - 1;
    // fused decode step whose token completes a block: warps 0 and 1 of group
    // 0 encode it (tail rows 0..R-2 and the new token) into archive slot
    // new_slot with the codec's own device code, so the archive is bitwise
    // what fc_append_step writes; the barrier publishes codes and scales to
    // the CTA
    if (last_chunk && a.step == 2) {
      if (grp == 0 && w < 2) encode_new_block<S, S * TPT>(a, w, lane, basis, b, h);
      ptx::named_bar_sync(kFinBar, 128 * NG);
    }
    // raw tail tokens, then the step's new token or block (last chunk)
    if (active && last_chunk && (a.nr > 0 || a.step != 0)) {
      float* red2 = reinterpret_cast<float*>(sm + C::xs) + grp * 4 * C::XW;
      // the raw tokens of the tail, and the step's new token, in one batch:
      // one reduction over the group for every logit, then one online-softmax
      // update (thread t = channel d)
      const int n_raw = a.step == 2 ? 0 : a.nr;  // a completed block is folded coded
      const int n_tok = n_raw + (a.step == 1 ? 1 : 0);
      constexpr int kTok = S * TPT;  // at most R tokens: R - 1 tail rows + the new one
      // every token's 32-bit words are requested first, before the query and
      // before any is used (a conversion right behind each load would wait
      // for it: one DRAM round trip per token), and converted where used
      const bool f32 = a.t_dtype == FC_DTYPE_F32;
      uint32_t kw[kTok], vw[kTok];
#pragma unroll
      for (int tt = 0; tt < kTok; ++tt) {
        kw[tt] = 0u;
        vw[tt] = 0u;
        if (tt < n_raw) {
          kw[tt] = __ldg(elem_word(a.kt, b * a.kts_b + h * a.kts_h + int64_t(tt) * kD + t, f32));
          vw[tt] = __ldg(elem_word(a.vt, b * a.vts_b + h * a.vts_h + int64_t(tt) * kD + t, f32));
        } else if (tt == n_raw && a.step == 1) {
          kw[tt] = __ldg(elem_word(a.kn, b * a.kns_b + h * a.kns_h + t, f32));
          vw[tt] = __ldg(elem_word(a.vn, b * a.vns_b + h * a.vns_h + t, f32));
        }
      }
      float qh[HPG];
#pragma unroll
      for (int y = 0; y < HPG; ++y) {
        const int g = min(grp + NG * y, G - 1);
        qh[y] = load_any(a.q, b * a.qs_b + (h * G + g) * a.qs_h + t, a.q_dtype) * a.qscale;
      }
      if (n_tok > 0) {
        // all R reductions at once (unused tokens hold zeros)
        float lgt[kTok][HPG];
#pragma unroll
        for (int tt = 0; tt < kTok; ++tt)
#pragma unroll
          for (int y = 0; y < HPG; ++y) lgt[tt][y] = warp_sum(qh[y] * word_elem(kw[tt], t, f32));
        if (lane == 0) {
#pragma unroll
          for (int tt = 0; tt < kTok; ++tt)
#pragma unroll
            for (int y = 0; y < HPG; ++y) red2[(w * kTok + tt) * HPG + y] = lgt[tt][y];
        }
        ptx::named_bar_sync(1 + grp, 128);
#pragma unroll
        for (int tt = 0; tt < kTok; ++tt)
#pragma unroll
          for (int y = 0; y < HPG; ++y)
            lgt[tt][y] = red2[(0 * kTok + tt) * HPG + y] + red2[(1 * kTok + tt) * HPG + y] +
                         red2[(2 * kTok + tt) * HPG + y] + red2[(3 * kTok + tt) * HPG + y];
        ptx::named_bar_sync(1 + grp, 128);  // red2 is reused below
#pragma unroll
        for (int y = 0; y < HPG; ++y) {
          float mn = Mh[y];
#pragma unroll
          for (int tt = 0; tt < kTok; ++tt)
            if (tt < n_tok) mn = fmaxf(mn, lgt[tt][y]);
          const float al = ptx::ex2(Mh[y] - mn);
          float ps = 0.f, add = 0.f;
#pragma unroll
          for (int tt = 0; tt < kTok; ++tt) {
            if (tt < n_tok) {
              const float p = ptx::ex2(lgt[tt][y] - mn);
              ps += p;
              add = fmaf(p, word_elem(vw[tt], t, f32), add);
            }
          }
          Ah[y] = fmaf(Ah[y], al, add);
          Lh[y] = fmaf(Lh[y], al, ps);
          Mh[y] = mn;
        }
      }
      if (a.step == 1 && grp == 0) {  // the token joins the tail at row nr
        copy_elem(a.kt, b * a.kts_b + h * a.kts_h + int64_t(a.nr) * kD + t, a.kn,
                  b * a.kns_b + h * a.kns_h + t, a.t_dtype);
        copy_elem(a.vt, b * a.vts_b + h * a.vts_h + int64_t(a.nr) * kD + t, a.vn,
                  b * a.vns_b + h * a.vns_h + t, a.t_dtype);
      }
      if (a.step == 2) {
        // the new block in the coefficient domain, as a tile row set would be:
        // s_j = scale_k,j C_k[j] . q, logits = A s, p, w = p A, acc += w scale_v C_v
        const StreamOut& ko = a.kout;
        const StreamOut& vo = a.vout;
        // (written by this CTA before the barrier above: read through L2)
        const signed char* kc = static_cast<const signed char*>(ko.coeffs) + b * ko.cs_b + h * ko.cs_h + a.new_slot * S * kD;
        const signed char* vc = static_cast<const signed char*>(vo.coeffs) + b * vo.cs_b + h * vo.cs_h + a.new_slot * S * kD;
        const float* ksp = ko.scales + b * ko.ss_b + h * ko.ss_h + a.new_slot * S;
        const float* vsp = vo.scales + b * vo.ss_b + h * vo.ss_h + a.new_slot * S;
        float ksc[S], vsc[S];
#pragma unroll
        for (int j = 0; j < S; ++j) {
          ksc[j] = __ldcg(ksp + j);
          vsc[j] = __ldcg(vsp + j);
        }
        int kcode[S], vraw[S];  // requested together, converted after
#pragma unroll
        for (int j = 0; j < S; ++j) {
          kcode[j] = __ldcg(kc + j * kD + t);
          vraw[j] = __ldcg(vc + j * kD + t);
        }
        float sj[S * HPG];
#pragma unroll
        for (int j = 0; j < S; ++j) {
          const float kv = float(kcode[j]);
#pragma unroll
          for (int y = 0; y < HPG; ++y) sj[j * HPG + y] = kv * qh[y];
        }
        group_sum<S * HPG>(sj, red2, w, lane, 1 + grp);
        float vcode[S];
#pragma unroll
        for (int j = 0; j < S; ++j) vcode[j] = float(vraw[j]);
#pragma unroll
        for (int y = 0; y < HPG; ++y) {
          float lg[S * TPT];
          float mx = Mh[y];
#pragma unroll
          for (int tk = 0; tk < S * TPT; ++tk) {
            float v = 0.f;
#pragma unroll
            for (int j = 0; j < S; ++j) v = fmaf(basis.m[j][tk], sj[j * HPG + y] * ksc[j], v);
            lg[tk] = v;
            mx = fmaxf(mx, v);
          }
          const float al = ptx::ex2(Mh[y] - mx);
          float ps = 0.f, wv[S];
#pragma unroll
          for (int j = 0; j < S; ++j) wv[j] = 0.f;
#pragma unroll
          for (int tk = 0; tk < S * TPT; ++tk) {
            const float p = ptx::ex2(lg[tk] - mx);
            ps += p;
#pragma unroll
            for (int j = 0; j < S; ++j) wv[j] = fmaf(p, basis.m[j][tk], wv[j]);
          }
          float add = 0.f;
#pragma unroll
          for (int j = 0; j < S; ++j) add = fmaf(wv[j] * vsc[j], vcode[j], add);
          Ah[y] = fmaf(Ah[y], al, add);
          Lh[y] = fmaf(Lh[y], al, ps);
          Mh[y] = mx;
        }
      }
    }
    if (active) {
#pragma unroll
      for (int y = 0; y < HPG; ++y) {
        const int g = grp + NG * y;
        if (g >= G) continue;
        const int hq = h * G + g;
        if (direct) {
          store_out(a.out, b * a.os_b + hq * a.os_h + t, a.out_dtype, Ah[y] / Lh[y]);
        } else {
          const int64_t row = (int64_t(b) * Hq + hq) * a.ns + c;
          a.pacc[row * kD + t] = Ah[y];
          if (t == 0) {
            a.pm[row] = Lh[y] > 0.f ? Mh[y] : -INFINITY;
            a.pl[row] = Lh[y];
          }
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  // every wait that can give up lies before the barrier above, so the abort
  // flag is final here (and the same for every thread). After an abort the
  // newest load of every stage lands and the last MMAs of each side complete
  // (a commit tracks all earlier MMAs of its thread) before the CTA frees
  // its TMEM and exits; older loads completed before their stage was reissued.
  if (*reinterpret_cast<volatile int*>(abort_flag)) {
    if (tma_warp && lane == 0) {
      for (int i = max(0, nk - NKS); i < nk; ++i) drain_wait(&kfull[i % NKS], uint32_t(i / NKS) & 1u);
      for (int i = max(0, nv - NVS); i < nv; ++i) drain_wait(&vfull[i % NVS], uint32_t(i / NVS) & 1u);
    }
    if (kmma_warp && lane == 0 && mk > 0) drain_wait(&kfree[(mk - 1) % NKS], uint32_t((mk - 1) / NKS) & 1u);
    if (vmma_warp && lane == 0 && mv > 0) drain_wait(&vfree[(mv - 1) % NVS], uint32_t((mv - 1) / NVS) & 1u);
    ptx::tc_fence_before();
    __syncthreads();
  }
  if (kmma_warp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }

  if (direct || !a.fuse) return;
  if (!last_cta_ticket(a.tickets + (b * a.Hk + h), ns_u, last_flag)) return;
  float* wts = reinterpret_cast<float*>(sm);  // the rings are free now
  const int64_t row = (int64_t(b) * Hq + h * G) * a.ns;
  combine_heads(a.pm + row, a.pl + row, a.pacc + row * kD, G, ns_u, a.ns, kD, wts, a.out,
                b * a.os_b + (h * G) * a.os_h, a.os_h, a.out_dtype);
  if (tid == 0) a.tickets[b * a.Hk + h] = 0u;
}

// ------------------------------------------------------------------ host

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::mutex mu;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// int8 codes of one archive as a 4-d tensor {D, live rows, H, B}, 128 x 128
// boxes with 128-byte swizzle
// Encoded tensor maps of recent archives, keyed by everything the encoding
// reads, so that a decode loop encodes each map once per archived block
// instead of once per launch (a small round-robin table, shared by host
// threads under a mutex).
struct MapKey {
  const void* base;
  int64_t rows, H, B, sh, sb, D;
  int kind;  // 2 S (codes) or 2 S + 1 (scales)
  bool operator==(const MapKey& o) const {
    return base == o.base && rows == o.rows && H == o.H && B == o.B && sh == o.sh && sb == o.sb &&
           D == o.D && kind == o.kind;
  }
};

template <typename Encode>
bool cached_map(CUtensorMap* m, const MapKey& key, Encode&& encode) {
  constexpr int kSlots = 32;
  static std::mutex mu;
  static MapKey keys[kSlots];
  static CUtensorMap maps[kSlots];
  static bool used[kSlots] = {false};
  static int next = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < kSlots; ++i)
      if (used[i] && keys[i] == key) {
        *m = maps[i];
        return true;
      }
  }
  if (!encode(m)) return false;
  std::lock_guard<std::mutex> lock(mu);
  keys[next] = key;
  maps[next] = *m;
  used[next] = true;
  next = (next + 1) % kSlots;
  return true;
}

bool encode_code_map(CUtensorMap* m, const fc_archive* arc, int64_t rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  const int64_t sh = arc->H > 1 ? arc->coeff_stride_h : arc->capacity * arc->S * arc->D;
  const int64_t sb = arc->B > 1 ? arc->coeff_stride_b : sh * arc->H;
  cuuint64_t dims[4] = {cuuint64_t(arc->D), cuuint64_t(rows), cuuint64_t(arc->H), cuuint64_t(arc->B)};
  cuuint64_t strides[3] = {cuuint64_t(arc->D), cuuint64_t(sh), cuuint64_t(sb)};
  cuuint32_t box[4] = {uint32_t(kD), uint32_t(kRows), 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, arc->coeffs, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 scales as a 3-d tensor {live rows, H, B}, boxes of 128 rows
bool encode_scale_map(CUtensorMap* m, const fc_archive* arc, int64_t rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  const int64_t sh = arc->H > 1 ? arc->scale_stride_h : arc->capacity * arc->S;
  const int64_t sb = arc->B > 1 ? arc->scale_stride_b : sh * arc->H;
  cuuint64_t dims[3] = {cuuint64_t(rows), cuuint64_t(arc->H), cuuint64_t(arc->B)};
  cuuint64_t strides[2] = {cuuint64_t(sh * 4), cuuint64_t(sb * 4)};
  cuuint32_t box[3] = {uint32_t(kRows), 1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, arc->scales, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_code_map(CUtensorMap* m, const fc_archive* arc, int64_t rows) {
  const MapKey key{arc->coeffs, rows, arc->H, arc->B, arc->H > 1 ? arc->coeff_stride_h : arc->capacity,
                   arc->B > 1 ? arc->coeff_stride_b : arc->capacity, arc->D, 2 * arc->S};
  return cached_map(m, key, [&](CUtensorMap* out) { return encode_code_map(out, arc, rows); });
}

bool make_scale_map(CUtensorMap* m, const fc_archive* arc, int64_t rows) {
  const MapKey key{arc->scales, rows, arc->H, arc->B, arc->H > 1 ? arc->scale_stride_h : arc->capacity,
                   arc->B > 1 ? arc->scale_stride_b : arc->capacity, arc->D, 2 * arc->S + 1};
  return cached_map(m, key, [&](CUtensorMap* out) { return encode_scale_map(out, arc, rows); });
}

// CTAs of one problem: every kv head takes ns chunks
int problem_ctas(const TcArgs& ta) { return ta.d.B * ta.d.Hk * ta.d.ns; }

template <int G, int S, int TPT, int NL>
int launch(const TcBatch<NL>& batch, const Basis& full, const BasisF64& full64, bool overlap,
           cudaStream_t stream) {
  TcBasis<S, S * TPT> basis;
  for (int j = 0; j < S; ++j)
    for (int t = 0; t < S * TPT; ++t) {
      basis.m[j][t] = full.m[j][t];
      basis.m64[j][t] = full64.m[j][t];
    }
  using C = Cfg<G, S, TPT>;
  const size_t smem = C::alloc;
  auto kern = decode_tc_kernel<G, S, TPT, NL>;
  // the attribute is a per-device property of the function: set once per
  // device (a launch on another device sets it there)
  static std::mutex attr_mu;
  static bool attr_set[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FC_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(attr_mu);
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
        return FC_ERR_CUDA;
      attr_set[dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(batch.cta_end[batch.n - 1]));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap ? 1 : 0;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, batch, basis));
}

// Fills problem slot i of a batch: the tile geometry and the four tensor maps.
template <int NL>
bool fill_problem(TcBatch<NL>* batch, int i, const DecodeArgs& d, const fc_archive* ka,
                  const fc_archive* va) {
  TcArgs& ta = batch->prob[i];
  ta.d = d;
  ta.tiles_per_head = tc_tiles_per_head(d.nb, d.S);
  ta.d.bal_q = d.ns;  // every kv head takes ns chunks
  ta.d.bal_rem = 0;
  const int64_t rows = d.nb * d.S;
  if (!make_code_map(&batch->maps[i][0], ka, rows) || !make_code_map(&batch->maps[i][1], va, rows) ||
      !make_scale_map(&batch->maps[i][2], ka, rows) || !make_scale_map(&batch->maps[i][3], va, rows))
    return false;
  batch->cta_end[i] = (i > 0 ? batch->cta_end[i - 1] : 0) + problem_ctas(ta);
  batch->n = i + 1;
  return true;
}

template <int NL>
int dispatch(const TcBatch<NL>& batch, int G, int S, int R, const Basis& basis, const BasisF64& basis64,
             bool overlap, cudaStream_t stream) {
  const int key = G * 10000 + S * 100 + R / S;
  switch (key) {
#define FC_TC_CASE(G, S, T) \
  case G * 10000 + S * 100 + T: return launch<G, S, T, NL>(batch, basis, basis64, overlap, stream);
    FC_TC_CASE(1, 1, 4) FC_TC_CASE(2, 1, 4) FC_TC_CASE(4, 1, 4) FC_TC_CASE(8, 1, 4)
    FC_TC_CASE(1, 1, 8) FC_TC_CASE(2, 1, 8) FC_TC_CASE(4, 1, 8)
    FC_TC_CASE(1, 2, 4) FC_TC_CASE(2, 2, 4) FC_TC_CASE(4, 2, 4) FC_TC_CASE(8, 2, 4)
    FC_TC_CASE(1, 2, 8) FC_TC_CASE(2, 2, 8) FC_TC_CASE(4, 2, 8)
    FC_TC_CASE(1, 4, 2) FC_TC_CASE(2, 4, 2) FC_TC_CASE(4, 4, 2) FC_TC_CASE(8, 4, 2)
    FC_TC_CASE(1, 4, 4) FC_TC_CASE(2, 4, 4) FC_TC_CASE(4, 4, 4) FC_TC_CASE(8, 4, 4)
    FC_TC_CASE(1, 8, 2) FC_TC_CASE(2, 8, 2) FC_TC_CASE(4, 8, 2) FC_TC_CASE(8, 8, 2)
#undef FC_TC_CASE
    default: return FC_ERR_UNSUPPORTED;
  }
}

}  // namespace tc

// Whether the tensor-core kernel serves this problem.
bool decode_tc_eligible(const fc_archive* ka, const fc_archive* va, int G) {
  if (ka->coeff_dtype != FC_DTYPE_I8 || va->coeff_dtype != FC_DTYPE_I8) return false;
  if (ka->codec != FC_CODEC_DCT || va->codec != FC_CODEC_DCT) return false;
  if (ka->D != tc::kD || ka->n_blocks < 1) return false;
  const int S = ka->S, R = ka->R;
  if (R % S) return false;
  const int tpt = R / S;
  if (!(G == 1 || G == 2 || G == 4 || G == 8)) return false;
  switch (S * 100 + tpt) {
    case 104: case 108: case 204: case 208: case 402: case 404: case 802: break;
    default: return false;
  }
  const int ni = G >= S ? G / S : 1;
  return ni * R <= 32;
}

int tc_tiles_per_head(int64_t nb, int S) { return int((nb + (tc::kRows / S) - 1) / (tc::kRows / S)); }

int launch_decode_tc(const DecodeArgs& d, const fc_archive* ka, const fc_archive* va, const Basis& basis,
                     cudaStream_t stream) {
  BasisF64 basis64;
  make_basis_f64(FC_CODEC_DCT, d.R, d.S, &basis64);
  tc::TcBatch<1> batch;
  if (!tc::fill_problem(&batch, 0, d, ka, va)) return FC_ERR_CUDA;
  return tc::dispatch(batch, d.G, d.S, d.R, basis, basis64, d.overlap != 0, stream);
}

int launch_decode_tc_layers(int n, const DecodeArgs* d, const fc_archive* const* ka, const fc_archive* const* va,
                            const Basis& basis, cudaStream_t stream) {
  if (n < 1 || n > FC_MAX_LAYERS) return FC_ERR_INVALID;
  BasisF64 basis64;
  make_basis_f64(FC_CODEC_DCT, d[0].R, d[0].S, &basis64);
  static_assert(FC_MAX_LAYERS == 16, "batch capacity");
  tc::TcBatch<FC_MAX_LAYERS> batch;
  for (int i = 0; i < n; ++i)
    if (!tc::fill_problem(&batch, i, d[i], ka[i], va[i])) return FC_ERR_CUDA;
  return tc::dispatch(batch, d[0].G, d[0].S, d[0].R, basis, basis64, d[0].overlap != 0, stream);
}

}  // namespace fc
