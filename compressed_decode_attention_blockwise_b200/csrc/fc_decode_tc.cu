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
// Warp roles. A TMA warp keeps a six-stage ring of 128-row tiles (K and V
// codes with 128-byte swizzle, plus their scales) full, refilling a stage as
// soon as the V-side MMA of its tile completes. Two MMA warps issue the K-side
// MMA of each tile as soon as it lands and the V-side MMA as soon as its W is
// written, so neither waits behind the other and both overlap the softmax. Up
// to four groups of four compute warps split the G query heads of the kv head;
// in a group, thread t owns coefficient row t on the K side and channel d = t
// on the V side, so every TMEM load is one warp quadrant. K sums are
// double-buffered and V sums triple-buffered in TMEM, W is triple-buffered in
// shared memory, and the V epilogue of tile i runs after the softmax of tile
// i+2.
// The online softmax keeps one running max per head for the CTA (one max per
// tile and group), each thread accumulates its own share of the softmax sum,
// and the output accumulator lives in registers (thread d, its group's heads).
//
// Every wait on an mbarrier is bounded; on timeout the kernel records an
// error in the workspace status word, stops issuing work, drains what it
// issued (also bounded), frees its TMEM and returns.
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "fc_decode.cuh"
#include "fc_tc_ptx.cuh"

namespace fc {
namespace tc {

constexpr int kRows = 128;  // coefficient rows per tile
constexpr int kD = 128;     // head dim served by this kernel
constexpr int kStages = 6;
constexpr uint32_t kTileBytes = kRows * kD;
constexpr uint32_t kStageTx = 2 * kTileBytes + 2 * kRows * 4;
constexpr unsigned long long kWaitCycles = 4000000000ull;  // ~2 s at 2 GHz

__host__ __device__ constexpr int pad8(int x) { return (x + 7) / 8 * 8; }
__host__ __device__ constexpr int pad16(int x) { return (x + 15) / 16 * 16; }

// Column layout of the MMA N dimension: GW groups of GH heads, each head three
// limb columns, each group padded to CS columns.
template <int G>
struct Cols {
  static constexpr int GW = G >= 4 ? 4 : G;  // compute warp groups (1, 2 or 4)
  static constexpr int GH = G / GW;          // heads per group
  static constexpr int CS = pad8(3 * GH);    // columns per group (8 or 16)
  static constexpr int NP = pad16(GW * CS);  // MMA N
  static constexpr int kComputeThreads = 128 * GW;
  static constexpr int kThreads = kComputeThreads + 96;  // + TMA, K-MMA and V-MMA warps
  // K sums double-buffered, V sums triple-buffered
  static constexpr uint32_t kTmemCols = 5 * NP <= 64 ? 64 : (5 * NP <= 128 ? 128 : 256);
};

struct TcArgs {
  DecodeArgs d;
  int tiles_per_head;
  int chunk_tiles;
};

template <int NP>
struct SmemLayout {
  static constexpr uint32_t k = 0;
  static constexpr uint32_t v = k + kStages * kTileBytes;
  static constexpr uint32_t qb = v + kStages * kTileBytes;   // K-major SW128, NP rows x 128 B
  static constexpr uint32_t wb = qb + NP * 128;               // 3 x (NP/16 x 128 rows x 16 B)
  static constexpr uint32_t ks = wb + 3 * NP * 128;
  static constexpr uint32_t vs = ks + kStages * kRows * 4;
  static constexpr uint32_t red = vs + kStages * kRows * 4;   // up to 4 groups x 4 warps x 32 floats
  static constexpr uint32_t bars = red + 4 * 4 * 32 * 4;
  // full[kStages], vdone[kStages], kfull[2], kempty[2], wready[3], vempty[3], qready
  static constexpr int kBars = 2 * kStages + 11;
  static constexpr uint32_t misc = bars + kBars * 8;          // tmem slot, abort, last
  static constexpr uint32_t bytes = misc + 16;
  static constexpr uint32_t alloc = bytes + 1024;             // alignment slack
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

// three 7-bit limbs of x in (-64, 64): x ~ L0 + L1 / 128 + L2 / 16384
__device__ __forceinline__ void limbs3(float x, int& l0, int& l1, int& l2) {
  l0 = __float2int_rn(x);
  const float r1 = (x - float(l0)) * 128.f;
  l1 = __float2int_rn(r1);
  const float r2 = (r1 - float(l1)) * 128.f;
  l2 = __float2int_rn(r2);
}

__device__ __forceinline__ float unlimb3(uint32_t c0, uint32_t c1, uint32_t c2) {
  return fmaf(float(int(c2)), 1.f / 16384.f, fmaf(float(int(c1)), 1.f / 128.f, float(int(c0))));
}

// byte offset of element (row n, column k) in a 128-byte-swizzled K-major
// operand whose rows are 128 bytes (1024-byte-aligned atoms of 8 rows)
__device__ __forceinline__ uint32_t sw128_offset(int n, int k) {
  return uint32_t(n) * 128u + ((uint32_t(k >> 4) ^ uint32_t(n & 7)) << 4) + uint32_t(k & 15);
}

struct Waiter {
  int* abort;
  uint32_t* status;
  __device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity) {
    if (*reinterpret_cast<volatile int*>(abort)) return false;
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = clock64();
    while (!ptx::mbar_try_wait(bar, parity)) {
      if (*reinterpret_cast<volatile int*>(abort)) return false;
      if (clock64() - t0 > kWaitCycles) {
        *reinterpret_cast<volatile int*>(abort) = 1;
        if (status) atomicOr(status, 1u);
        return false;
      }
    }
    return true;
  }
};

// Sums G values per thread over the 128 threads of one warp group (named
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

template <int CS>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[CS]) {
  if constexpr (CS == 8) {
    ptx::tmem_ld8(taddr, r);
  } else {
    ptx::tmem_ld16(taddr, r);
  }
}

template <int G, int S, int TPT>
__global__ void __launch_bounds__(Cols<G>::kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                     const TcArgs ta, const Basis basis) {
  using C = Cols<G>;
  constexpr int GW = C::GW, GH = C::GH, CS = C::CS, NP = C::NP;
  constexpr int NCT = C::kComputeThreads;
  constexpr int R = S * TPT;
  constexpr int TB = kRows / S;  // blocks per tile
  using L = SmemLayout<NP>;
  static_assert(kRows % S == 0 && 32 % S == 0, "blocks must not straddle warps");
  static_assert(NP == 16 || NP == 32, "N must be 16 or 32");
  static_assert(GH % 2 == 0 || GH == 1, "heads per group pair up");
  constexpr uint32_t kIdescK = ptx::idesc_i8(128, NP, false, false);
  constexpr uint32_t kIdescV = ptx::idesc_i8(128, NP, true, true);
  constexpr uint32_t kWBytes = NP * 128;  // one W buffer

  const DecodeArgs& a = ta.d;
  extern __shared__ uint8_t smem_raw[];
  // 128-byte swizzle atoms need 1024-byte alignment in the shared window
  uint8_t* sm = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::bars);
  uint64_t* full = bars;               // tile landed (TMA -> MMA)
  uint64_t* vdone = bars + kStages;    // V-side MMA of the stage's tile done (-> compute, TMA)
  uint64_t* kfull = bars + 2 * kStages;
  uint64_t* kempty = kfull + 2;
  uint64_t* wready = kfull + 4;        // 3 W buffers
  uint64_t* vempty = kfull + 7;        // 3 V accumulators
  uint64_t* qready = kfull + 10;       // query limbs written (compute -> MMA)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::misc);
  int* abort_flag = reinterpret_cast<int*>(sm + L::misc + 4);
  int* last_flag = reinterpret_cast<int*>(sm + L::misc + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int Hq = a.Hk * G;
  Waiter waiter{abort_flag, a.status};

  const int tile0 = c * ta.chunk_tiles;
  const int tile1 = min(tile0 + ta.chunk_tiles, ta.tiles_per_head);
  const int ntiles = max(0, tile1 - tile0);
  const bool producer = warp >= NCT / 32;  // TMA warp, K-MMA warp, V-MMA warp
  const bool tma_warp = warp == NCT / 32;
  const bool mma_warp = warp == NCT / 32 + 1;   // K side; also owns the TMEM allocation
  const bool mmav_warp = warp == NCT / 32 + 2;  // V side

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&vdone[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&kfull[i], 1);
      ptx::mbar_init(&kempty[i], NCT);
    }
    for (int i = 0; i < 3; ++i) {
      ptx::mbar_init(&wready[i], NCT);
      ptx::mbar_init(&vempty[i], NCT);
    }
    ptx::mbar_init(qready, NCT);
    *abort_flag = 0;
    *last_flag = 0;
    ptx::fence_mbar_init();
  }
  if (mma_warp) {
    ptx::tmem_alloc(tmem_slot, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  if (tma_warp) {
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_k);
      ptx::prefetch_tmap(&tm_v);
      ptx::prefetch_tmap(&tm_ks);
      ptx::prefetch_tmap(&tm_vs);
    }
  }

  // barriers and the TMEM address are visible to every warp from here on; the
  // TMA warp starts streaming while the compute warps prepare the query limbs
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // compute-thread identity: group gw, thread t in the group (row / channel)
  const int gw = producer ? 0 : tid / 128;
  const int t = tid & 127;
  const int wq = warp & 3;  // TMEM lane quadrant of this warp
  const int g0 = gw * GH;   // first head of my group
  const int bar_id = 1 + gw;
  float* red = reinterpret_cast<float*>(sm + L::red) + gw * 128;

  // ---- query limbs: thread t = channel d, heads of its group
  float qd[GH];
  float qunit[GH];  // 2^(E_q - 6): weight of limb 0
  if (!producer) {
#pragma unroll
    for (int i = 0; i < GH; ++i)
      qd[i] = load_any(a.q, b * a.qs_b + (h * G + g0 + i) * a.qs_h + t, a.q_dtype) * a.qscale;
    float qmax[GH];
#pragma unroll
    for (int i = 0; i < GH; ++i) qmax[i] = warp_max(fabsf(qd[i]));
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < GH; ++i) red[wq * 32 + i] = qmax[i];
    }
    ptx::named_bar_sync(bar_id, 128);
    uint8_t* qb = sm + L::qb;
#pragma unroll
    for (int i = 0; i < GH; ++i) {
      const float mx = fmaxf(fmaxf(red[i], red[32 + i]), fmaxf(red[64 + i], red[96 + i]));
      const int e = exp_above(mx);
      qunit[i] = pow2i(e - 6);
      int l0, l1, l2;
      limbs3(qd[i] * pow2i(6 - e), l0, l1, l2);
      const int n = gw * CS + 3 * i;
      qb[sw128_offset(n + 0, t)] = static_cast<uint8_t>(l0);
      qb[sw128_offset(n + 1, t)] = static_cast<uint8_t>(l1);
      qb[sw128_offset(n + 2, t)] = static_cast<uint8_t>(l2);
    }
    for (int n = gw * CS + 3 * GH; n < (gw + 1) * CS; ++n) qb[sw128_offset(n, t)] = 0;
    if (gw == GW - 1)
      for (int n = GW * CS; n < NP; ++n) qb[sw128_offset(n, t)] = 0;
    ptx::fence_proxy_async_smem();
    ptx::mbar_arrive(qready);
  }
  if (tma_warp && lane == 0) {
    // ================= TMA warp: keep the ring full. Stage s is refilled as
    // soon as the V-side MMA of the tile it held has completed.
    int loaded = 0;
    for (; loaded < ntiles; ++loaded) {
      const int s = loaded % kStages;
      if (loaded >= kStages) waiter.wait(&vdone[s], uint32_t(loaded / kStages - 1) & 1u);
      if (*reinterpret_cast<volatile int*>(abort_flag)) break;
      const int row0 = (tile0 + loaded) * kRows;
      ptx::mbar_arrive_expect_tx(&full[s], kStageTx);
      ptx::tma_load_4d(sm + L::k + s * kTileBytes, &tm_k, &full[s], 0, row0, h, b);
      ptx::tma_load_4d(sm + L::v + s * kTileBytes, &tm_v, &full[s], 0, row0, h, b);
      ptx::tma_load_3d(sm + L::ks + s * kRows * 4, &tm_ks, &full[s], row0, h, b);
      ptx::tma_load_3d(sm + L::vs + s * kRows * 4, &tm_vs, &full[s], row0, h, b);
    }
    // after an abort, every issued load must land before the CTA exits (bounded)
    if (*reinterpret_cast<volatile int*>(abort_flag)) {
      const unsigned long long t0 = clock64();
      for (int i = 0; i < loaded; ++i)
        while (!ptx::mbar_try_wait(&full[i % kStages], uint32_t(i / kStages) & 1u) &&
               clock64() - t0 < kWaitCycles) {
        }
    }
  }
  if (mma_warp && lane == 0) {
    // ================= K-MMA warp: S_int of each tile as soon as it lands
    waiter.wait(qready, 0u);
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % kStages, bb = i & 1;
      waiter.wait(&full[s], uint32_t(i / kStages) & 1u);
      waiter.wait(&kempty[bb], (uint32_t(i >> 1) & 1u) ^ 1u);
      if (*reinterpret_cast<volatile int*>(abort_flag)) break;
      ptx::tc_fence_after();
      const uint32_t ka = ptx::smem_u32(sm + L::k + s * kTileBytes);
      const uint32_t qa = ptx::smem_u32(sm + L::qb);
#pragma unroll
      for (int k = 0; k < kD / 32; ++k)
        ptx::mma_i8(tmem + bb * NP, ptx::desc_sw128(ka + 32 * k, 16, 1024),
                    ptx::desc_sw128(qa + 32 * k, 16, 1024), kIdescK, k > 0 ? 1u : 0u);
      ptx::mma_commit(&kfull[bb]);
    }
  }
  if (mmav_warp && lane == 0) {
    // ================= V-MMA warp: Acc_int of each tile as soon as its W is ready
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % kStages, vb = i % 3;
      waiter.wait(&wready[vb], uint32_t(i / 3) & 1u);
      waiter.wait(&vempty[vb], (uint32_t(i / 3) & 1u) ^ 1u);
      if (*reinterpret_cast<volatile int*>(abort_flag)) break;
      ptx::tc_fence_after();
      const uint32_t va = ptx::smem_u32(sm + L::v + s * kTileBytes);
      const uint32_t wa = ptx::smem_u32(sm + L::wb + vb * kWBytes);
#pragma unroll
      for (int k = 0; k < kRows / 32; ++k)
        ptx::mma_i8(tmem + 2 * NP + vb * NP, ptx::desc_sw128(va + 4096 * k, kTileBytes, 1024),
                    ptx::desc_noswizzle(wa + 512 * k, 128, 2048), kIdescV, k > 0 ? 1u : 0u);
      // completes when this and every earlier V-side MMA has finished; the
      // K-side MMA of the same tile finished before its W could be written
      ptx::mma_commit(&vdone[s]);
    }
  }

  // ================= compute warps
  float m_run[GH], lsum[GH], acc[GH];
#pragma unroll
  for (int i = 0; i < GH; ++i) {
    m_run[i] = -INFINITY;
    lsum[i] = 0.f;
    acc[i] = 0.f;
  }
  if (!producer) {
    const int j = lane % S;
    float2 areg[TPT][S];  // (A[t][jj], A[t][jj]) for my tokens t = j * TPT + i
#pragma unroll
    for (int i = 0; i < TPT; ++i)
#pragma unroll
      for (int jj = 0; jj < S; ++jj) {
        const float av = basis.m[jj][j * TPT + i];
        areg[i][jj] = make_float2(av, av);
      }
    const float sqrtR = sqrtf(float(R));
    const uint32_t lane_off = uint32_t(wq * 32) << 16;
    const uint32_t col0 = uint32_t(gw * CS);
    // softmax rescale and W unit of the two tiles whose V epilogue is pending
    float alpha_p1[GH], wunit_p1[GH], alpha_p2[GH], wunit_p2[GH];
#pragma unroll
    for (int i = 0; i < GH; ++i) {
      alpha_p1[i] = alpha_p2[i] = 1.f;
      wunit_p1[i] = wunit_p2[i] = 0.f;
    }

    // V epilogue of tile i: acc = alpha(i) acc + W-limb sums (run two tiles
    // late, so the V-side MMA round trip overlaps two softmax passes)
    auto v_epilogue = [&](int i, const float (&al)[GH], const float (&wu)[GH]) {
      const int vb = i % 3;
      waiter.wait(&vdone[i % kStages], uint32_t(i / kStages) & 1u);
      ptx::tc_fence_after();
      uint32_t vr[CS];
      tmem_ld_cols<CS>(tmem + 2 * NP + vb * NP + col0 + lane_off, vr);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&vempty[vb]);
#pragma unroll
      for (int g = 0; g < GH; ++g)
        acc[g] = fmaf(acc[g], al[g], wu[g] * unlimb3(vr[3 * g], vr[3 * g + 1], vr[3 * g + 2]));
    };

    for (int it = 0; it < ntiles; ++it) {
      const int s = it % kStages, bb = it & 1;
      const int tile = tile0 + it;
      // ---- K side results
      waiter.wait(&kfull[bb], uint32_t(it >> 1) & 1u);
      ptx::tc_fence_after();
      uint32_t cr[CS];
      tmem_ld_cols<CS>(tmem + bb * NP + col0 + lane_off, cr);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      ptx::mbar_arrive(&kempty[bb]);
      const float sk = reinterpret_cast<const float*>(sm + L::ks)[s * kRows + t];
      const float sv = reinterpret_cast<const float*>(sm + L::vs)[s * kRows + t];
      float sval[GH];
#pragma unroll
      for (int g = 0; g < GH; ++g) sval[g] = sk * qunit[g] * unlimb3(cr[3 * g], cr[3 * g + 1], cr[3 * g + 2]);

      // gather the S rows of my block
      float sb[S][GH];
#pragma unroll
      for (int jj = 0; jj < S; ++jj)
#pragma unroll
        for (int g = 0; g < GH; ++g) sb[jj][g] = __shfl_sync(0xffffffffu, sval[g], (lane - j) + jj);

      const bool live = int64_t(tile) * TB + t / S < a.nb;
      // logits of my TPT tokens, heads in pairs (packed fp32x2 FMA)
      float lg[TPT][GH];
#pragma unroll
      for (int i = 0; i < TPT; ++i) {
        if constexpr (GH == 1) {
          float x = 0.f;
#pragma unroll
          for (int jj = 0; jj < S; ++jj) x = fmaf(areg[i][jj].x, sb[jj][0], x);
          lg[i][0] = x;
        } else {
#pragma unroll
          for (int g = 0; g < GH; g += 2) {
            float2 x = make_float2(0.f, 0.f);
#pragma unroll
            for (int jj = 0; jj < S; ++jj) x = __ffma2_rn(areg[i][jj], make_float2(sb[jj][g], sb[jj][g + 1]), x);
            lg[i][g] = x.x;
            lg[i][g + 1] = x.y;
          }
        }
      }
      float tmax[GH];
#pragma unroll
      for (int g = 0; g < GH; ++g) {
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < TPT; ++i) mx = fmaxf(mx, lg[i][g]);
        tmax[g] = live ? mx : -INFINITY;
      }
      // tile-wide max per head and the largest V scale of the tile
      float vmax = sv;
#pragma unroll
      for (int g = 0; g < GH; ++g) tmax[g] = warp_max(tmax[g]);
      vmax = warp_max(vmax);
      if (lane == 0) {
#pragma unroll
        for (int g = 0; g < GH; ++g) red[wq * 32 + g] = tmax[g];
        red[wq * 32 + 31] = vmax;
      }
      ptx::named_bar_sync(bar_id, 128);
#pragma unroll
      for (int g = 0; g < GH; ++g) tmax[g] = fmaxf(fmaxf(red[g], red[32 + g]), fmaxf(red[64 + g], red[96 + g]));
      vmax = fmaxf(fmaxf(red[31], red[63]), fmaxf(red[95], red[127]));
      ptx::named_bar_sync(bar_id, 128);  // red is rewritten next tile

      float m_new[GH], alpha[GH], wunit[GH], winv[GH];
#pragma unroll
      for (int g = 0; g < GH; ++g) {
        m_new[g] = fmaxf(m_run[g], tmax[g]);
        alpha[g] = ptx::ex2(m_run[g] - m_new[g]);
        const int e = exp_above(ptx::ex2(tmax[g] - m_new[g]) * sqrtR * vmax);
        wunit[g] = pow2i(e - 6);
        winv[g] = pow2i(6 - e);
      }
      // p, the softmax sum, and my tokens' share of w_jj = sum_t p_t A[t][jj]
      float2 wpart[S][(GH + 1) / 2];
#pragma unroll
      for (int jj = 0; jj < S; ++jj)
#pragma unroll
        for (int g2 = 0; g2 < (GH + 1) / 2; ++g2) wpart[jj][g2] = make_float2(0.f, 0.f);
      float ps[GH];
#pragma unroll
      for (int g = 0; g < GH; ++g) ps[g] = 0.f;
#pragma unroll
      for (int i = 0; i < TPT; ++i) {
        float p[GH];
#pragma unroll
        for (int g = 0; g < GH; ++g) {
          p[g] = live ? ptx::ex2(lg[i][g] - m_new[g]) : 0.f;
          ps[g] += p[g];
        }
        if constexpr (GH == 1) {
#pragma unroll
          for (int jj = 0; jj < S; ++jj) wpart[jj][0].x = fmaf(p[0], areg[i][jj].x, wpart[jj][0].x);
        } else {
#pragma unroll
          for (int g = 0; g < GH; g += 2)
#pragma unroll
            for (int jj = 0; jj < S; ++jj)
              wpart[jj][g / 2] = __ffma2_rn(make_float2(p[g], p[g + 1]), areg[i][jj], wpart[jj][g / 2]);
        }
      }
#pragma unroll
      for (int g = 0; g < GH; ++g) lsum[g] = fmaf(lsum[g], alpha[g], ps[g]);
      // sum the shares over the S lanes of the block
#pragma unroll
      for (int o = 1; o < S; o <<= 1)
#pragma unroll
        for (int jj = 0; jj < S; ++jj)
#pragma unroll
          for (int g2 = 0; g2 < (GH + 1) / 2; ++g2) {
            float2 other;
            other.x = __shfl_xor_sync(0xffffffffu, wpart[jj][g2].x, o);
            other.y = GH == 1 ? 0.f : __shfl_xor_sync(0xffffffffu, wpart[jj][g2].y, o);
            wpart[jj][g2] = __fadd2_rn(wpart[jj][g2], other);
          }
      // W = w_j * scale_v as three int8 limbs: this group's CS bytes of row t
      {
        uint32_t packed[CS / 4];
#pragma unroll
        for (int q = 0; q < CS / 4; ++q) packed[q] = 0u;
#pragma unroll
        for (int g = 0; g < GH; ++g) {
          float wj = 0.f;
#pragma unroll
          for (int jj = 0; jj < S; ++jj) {
            const float cand = (g & 1) ? wpart[jj][g / 2].y : wpart[jj][g / 2].x;
            wj = (jj == j) ? cand : wj;
          }
          int l[3];
          limbs3(wj * sv * winv[g], l[0], l[1], l[2]);
#pragma unroll
          for (int k = 0; k < 3; ++k) {
            const int byte = 3 * g + k;
            packed[byte / 4] |= (uint32_t(l[k]) & 0xffu) << (8 * (byte % 4));
          }
        }
        uint8_t* wrow = sm + L::wb + (it % 3) * kWBytes;
        // column c of row t lives at (c / 16) * 2048 + t * 16 + c % 16
        if constexpr (CS == 8) {
          *reinterpret_cast<uint2*>(wrow + (gw / 2) * 2048 + t * 16 + (gw % 2) * 8) =
              make_uint2(packed[0], packed[1]);
        } else {
          *reinterpret_cast<uint4*>(wrow + gw * 2048 + t * 16) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(&wready[it % 3]);
#pragma unroll
      for (int g = 0; g < GH; ++g) m_run[g] = m_new[g];

      // ---- V epilogue of the tile two back (its MMA overlapped two softmaxes)
      if (it >= 2) v_epilogue(it - 2, alpha_p2, wunit_p2);
#pragma unroll
      for (int g = 0; g < GH; ++g) {
        alpha_p2[g] = alpha_p1[g];
        wunit_p2[g] = wunit_p1[g];
        alpha_p1[g] = alpha[g];
        wunit_p1[g] = wunit[g];
      }
    }
    if (ntiles >= 2) v_epilogue(ntiles - 2, alpha_p2, wunit_p2);
    if (ntiles >= 1) v_epilogue(ntiles - 1, alpha_p1, wunit_p1);

    // ---- raw tail tokens (last chunk): thread t = channel d
    if (c == a.ns - 1) {
      for (int tt = 0; tt < a.nr; ++tt) {
        const float kd = load_any(a.kt, b * a.kts_b + h * a.kts_h + int64_t(tt) * kD + t, a.t_dtype);
        const float vd = load_any(a.vt, b * a.vts_b + h * a.vts_h + int64_t(tt) * kD + t, a.t_dtype);
        float lgt[GH];
#pragma unroll
        for (int g = 0; g < GH; ++g) lgt[g] = qd[g] * kd;
        group_sum<GH>(lgt, red, wq, lane, bar_id);
#pragma unroll
        for (int g = 0; g < GH; ++g) {
          const float mn = fmaxf(m_run[g], lgt[g]);
          const float al = ptx::ex2(m_run[g] - mn);
          const float p = ptx::ex2(lgt[g] - mn);
          acc[g] = fmaf(acc[g], al, p * vd);
          lsum[g] = fmaf(lsum[g], al, t == 0 ? p : 0.f);
          m_run[g] = mn;
        }
      }
    }
    group_sum<GH>(lsum, red, wq, lane, bar_id);
  }

  // ---- partials (or the output)
  const bool direct = a.fuse && a.ns == 1;
  if (!producer) {
#pragma unroll
    for (int g = 0; g < GH; ++g) {
      const int hq = h * G + g0 + g;
      if (direct) {
        store_out(a.out, b * a.os_b + hq * a.os_h + t, a.out_dtype, acc[g] / lsum[g]);
      } else {
        const int64_t row = (int64_t(b) * Hq + hq) * a.ns + c;
        a.pacc[row * kD + t] = acc[g];
        if (t == 0) {
          a.pm[row] = lsum[g] > 0.f ? m_run[g] : -INFINITY;
          a.pl[row] = lsum[g];
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (mma_warp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }

  if (direct || !a.fuse) return;
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned tk = atomicAdd(a.tickets + (b * a.Hk + h), 1u);
    *last_flag = (tk == unsigned(a.ns - 1)) ? 1 : 0;
  }
  __syncthreads();
  if (!*last_flag) return;
  __threadfence();
  float* wts = reinterpret_cast<float*>(sm);  // stage buffers are free now
  const int64_t row = (int64_t(b) * Hq + h * G) * a.ns;
  combine_heads(a.pm + row, a.pl + row, a.pacc + row * kD, G, a.ns, kD, wts, a.out,
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
bool make_code_map(CUtensorMap* m, const fc_archive* arc, int64_t rows) {
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
bool make_scale_map(CUtensorMap* m, const fc_archive* arc, int64_t rows) {
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

template <int G, int S, int TPT>
int launch(const TcArgs& ta, const Basis& basis, const CUtensorMap* maps, cudaStream_t stream) {
  using Cl = Cols<G>;
  const size_t smem = SmemLayout<Cl::NP>::alloc;
  auto kern = decode_tc_kernel<G, S, TPT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return FC_ERR_CUDA;
  const dim3 grid(unsigned(ta.d.ns), unsigned(ta.d.Hk), unsigned(ta.d.B));
  kern<<<grid, Cl::kThreads, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], ta, basis);
  return cuda_status(cudaGetLastError());
}

}  // namespace tc

// Whether the tensor-core kernel serves this problem.
bool decode_tc_eligible(const fc_archive* ka, const fc_archive* va, int G) {
  if (ka->coeff_dtype != FC_DTYPE_I8 || va->coeff_dtype != FC_DTYPE_I8) return false;
  if (ka->D != tc::kD || ka->n_blocks < 1) return false;
  const int S = ka->S, R = ka->R;
  if (R % S) return false;
  const int tpt = R / S;
  if (!(G == 1 || G == 2 || G == 4 || G == 8)) return false;
  switch (S * 100 + tpt) {
    case 204: case 208: case 402: case 404: case 802: case 104: case 108: break;
    default: return false;
  }
  return S * G <= 32 && tpt * G <= 32;
}

int tc_tiles_per_head(int64_t nb, int S) { return int((nb + (tc::kRows / S) - 1) / (tc::kRows / S)); }

int launch_decode_tc(const DecodeArgs& d, const fc_archive* ka, const fc_archive* va, const Basis& basis,
                     cudaStream_t stream) {
  tc::TcArgs ta;
  ta.d = d;
  ta.tiles_per_head = tc_tiles_per_head(d.nb, d.S);
  ta.chunk_tiles = (ta.tiles_per_head + d.ns - 1) / d.ns;
  CUtensorMap maps[4];
  const int64_t rows = d.nb * d.S;
  if (!tc::make_code_map(&maps[0], ka, rows) || !tc::make_code_map(&maps[1], va, rows) ||
      !tc::make_scale_map(&maps[2], ka, rows) || !tc::make_scale_map(&maps[3], va, rows))
    return FC_ERR_CUDA;
  const int key = d.G * 10000 + d.S * 100 + d.R / d.S;
  switch (key) {
#define FC_TC_CASE(G, S, T) \
  case G * 10000 + S * 100 + T: return tc::launch<G, S, T>(ta, basis, maps, stream);
    FC_TC_CASE(1, 2, 4) FC_TC_CASE(2, 2, 4) FC_TC_CASE(4, 2, 4) FC_TC_CASE(8, 2, 4)
    FC_TC_CASE(1, 2, 8) FC_TC_CASE(2, 2, 8) FC_TC_CASE(4, 2, 8)
    FC_TC_CASE(1, 4, 2) FC_TC_CASE(2, 4, 2) FC_TC_CASE(4, 4, 2) FC_TC_CASE(8, 4, 2)
    FC_TC_CASE(1, 4, 4) FC_TC_CASE(2, 4, 4) FC_TC_CASE(4, 4, 4) FC_TC_CASE(8, 4, 4)
    FC_TC_CASE(1, 8, 2) FC_TC_CASE(2, 8, 2) FC_TC_CASE(4, 8, 2)
    FC_TC_CASE(1, 1, 4) FC_TC_CASE(2, 1, 4) FC_TC_CASE(4, 1, 4) FC_TC_CASE(8, 1, 4)
    FC_TC_CASE(1, 1, 8) FC_TC_CASE(2, 1, 8) FC_TC_CASE(4, 1, 8)
#undef FC_TC_CASE
    default: return FC_ERR_UNSUPPORTED;
  }
}

}  // namespace fc
