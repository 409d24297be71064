// Coefficient-domain decode attention: split-K partials, the CTA-level merge,
// and the combine (shared by the fused last-CTA path and fc_combine).
//
// flashcodec/triton_attention.py (module docstring, split kernel) and the
// flashcodec-kv README, "Materialization-free decode attention": the R tokens
// of a block are K_blk = A C_k with A = M^T (R x S), so a decode query scores a
// whole block from its S coefficient rows:
//   s = C_k q            (S values, one dot product of length D per row)
//   logits = sigma A s   (R values)
//   online softmax       m' = max(m, max logits), p = e^(logits - m'),
//                        alpha = e^(m - m'), l = alpha l + sum p
//   w = p A              (S values)
//   acc = alpha acc + w C_v
// The raw tail tokens enter the same softmax one at a time; the last chunk of
// the split owns them. Chunk partials (m, l, acc) merge with the usual
// max-rescale (combine kernel).
//
// This file holds the portable CUDA-core kernel that serves every supported
// dtype combination: one CTA of 4 warps per (chunk, kv head, batch); each
// warp walks every 4th block of the chunk with its own softmax state; lane l
// owns channels [l * VEC, (l + 1) * VEC) of q and acc for all G query heads of
// the kv head, so every coefficient byte is read once per kv head and shared by
// the whole GQA group. q is pre-multiplied by sigma * log2(e) and the softmax
// runs in base 2 (exp2), which leaves every ratio of exponentials unchanged.
#pragma once

#include <type_traits>

#include "fc_encode.cuh"

namespace fc {

constexpr int kMaxSplits = 512;
constexpr int kGenericWarps = 4;

struct DecodeArgs {
  const void* q;
  int q_dtype;
  int64_t qs_b, qs_h;
  const void* kc;
  const float* ks;
  int64_t kcs_b, kcs_h, kss_b, kss_h;
  const void* vc;
  const float* vs;
  int64_t vcs_b, vcs_h, vss_b, vss_h;
  const void* kt;
  const void* vt;
  int t_dtype;
  int64_t kts_b, kts_h, vts_b, vts_h;
  int nr;  // live tail tokens
  int B, Hk, G, R, S, D;
  int64_t nb;
  int ns;         // split slots per (b, q head) in the workspace
  int64_t chunk;
  // tensor-core kernel, automatic split: the first bal_rem kv heads take
  // bal_q + 1 chunks, the others bal_q (one CTA per SM in all); 0 = ns each
  int bal_q, bal_rem;
  int auto_split;  // num_splits was 0: ns is the planner's slot count
  int test_stall;  // test hook: one wait that nothing ends, with a short limit
  float qscale;  // sigma * log2(e)
  uint32_t* status;
  uint32_t* tickets;
  float* pm;
  float* pl;
  float* pacc;
  int fuse;     // 1: last CTA per kv head writes out
  int overlap;  // 1: launched as a programmatic dependent (FC_DECODE_OVERLAP)
  int q_final;  // 1: q may be read before the dependency wait (FC_DECODE_Q_FINAL)
  // fused decode step (fc_decode_step): 0 plain attention; 1 the new token
  // joins the tail at row nr; 2 it completes the block formed by the nr = R - 1
  // tail rows, which is encoded into archive slot new_slot (= nb)
  int step;
  const void* kn;
  const void* vn;
  int64_t kns_b, kns_h, vns_b, vns_h;
  StreamOut kout, vout;
  int64_t new_slot;
  void* out;
  int out_dtype;
  int64_t os_b, os_h;
};

__device__ __forceinline__ void store_out(void* out, int64_t idx, int dtype, float v) {
  if (dtype == FC_DTYPE_F32)
    static_cast<float*>(out)[idx] = v;
  else
    static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
}

// Merges the ns split partials of NH consecutive query heads into their
// outputs: M = max_c m_c, L = sum_c l_c e^(m_c - M), out = sum_c acc_c
// e^(m_c - M) / L, chunks with l_c = 0 skipped (base-2 exponentials: the
// partial maxima are kept in log2 units). Head i's partials are rows
// pm[i * stride + c], pl[i * stride + c], pacc[(i * stride + c) * D + d]
// (stride >= ns: the workspace's split slots per head); its output goes to
// out[out_off + i * out_stride_h + d]. All threads of the CTA take part. Each
// thread first issues the loads of the partial accumulators of its first
// (head, channel) output (up to kPre of them) and only then do warps compute
// the per-head weights into shared scratch `wts` (NH * (ns + 1) floats), so
// both sets of L2 reads are in flight together; further outputs (more outputs
// than threads) and partials beyond kPre use batched loads. Partials written
// by other CTAs of the same launch are read through L2 (ld.cg).
__device__ __forceinline__ void combine_heads(const float* pm, const float* pl, const float* pacc, int NH,
                                              int ns, int stride, int D, float* wts, void* out,
                                              int64_t out_off, int64_t out_stride_h, int out_dtype) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int n_out = NH * D;
  constexpr int kPre = 24;
  // partials of my first output, requested before the weights are known
  const bool has_first = tid < n_out;
  const int fi = has_first ? tid / D : 0, fd = has_first ? tid - fi * D : 0;
  const float* fsrc = pacc + int64_t(fi) * stride * D + fd;
  float pre[kPre];
#pragma unroll
  for (int u = 0; u < kPre; ++u) pre[u] = (has_first && u < ns) ? __ldcg(fsrc + int64_t(u) * D) : 0.f;

  constexpr int kReg = 4;  // partial rows per lane kept in registers (ns <= 128)
  for (int i = warp; i < NH; i += nwarps) {
    const float* m = pm + int64_t(i) * stride;
    const float* l = pl + int64_t(i) * stride;
    float* w = wts + i * (ns + 1);
    float mx = -INFINITY, L = 0.f;
    if (ns <= 32 * kReg) {
      float mv[kReg], lv[kReg];
#pragma unroll
      for (int r = 0; r < kReg; ++r) {
        const int c = lane + 32 * r;
        mv[r] = c < ns ? __ldcg(m + c) : -INFINITY;
        lv[r] = c < ns ? __ldcg(l + c) : 0.f;
      }
#pragma unroll
      for (int r = 0; r < kReg; ++r)
        if (lv[r] > 0.f) mx = fmaxf(mx, mv[r]);
      mx = warp_max(mx);
#pragma unroll
      for (int r = 0; r < kReg; ++r) {
        const int c = lane + 32 * r;
        const float e = lv[r] > 0.f ? exp2f(mv[r] - mx) : 0.f;
        if (c < ns) w[c] = e;
        L = fmaf(lv[r], e, L);
      }
    } else {
      for (int c = lane; c < ns; c += 32)
        if (__ldcg(l + c) > 0.f) mx = fmaxf(mx, __ldcg(m + c));
      mx = warp_max(mx);
      for (int c = lane; c < ns; c += 32) {
        const float lc = __ldcg(l + c);
        const float e = lc > 0.f ? exp2f(__ldcg(m + c) - mx) : 0.f;
        w[c] = e;
        L = fmaf(lc, e, L);
      }
    }
    L = warp_sum(L);
    if (lane == 0) w[ns] = 1.f / L;
  }
  __syncthreads();
  if (has_first) {
    const float* w = wts + fi * (ns + 1);
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < kPre; ++u)
      if (u < ns) acc = fmaf(pre[u], w[u], acc);
    for (int c = kPre; c < ns; ++c) acc = fmaf(__ldcg(fsrc + int64_t(c) * D), w[c], acc);
    store_out(out, out_off + fi * out_stride_h + fd, out_dtype, acc * w[ns]);
  }
  // the remaining outputs, 16 partials in flight at a time
  for (int o = tid + blockDim.x; o < n_out; o += blockDim.x) {
    const int i = o / D, d = o - i * D;
    const float* w = wts + i * (ns + 1);
    const float* src = pacc + int64_t(i) * stride * D + d;
    float acc = 0.f;
    for (int c0 = 0; c0 < ns; c0 += 16) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = c0 + u < ns ? __ldcg(src + int64_t(c0 + u) * D) : 0.f;
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (c0 + u < ns) acc = fmaf(v[u], w[c0 + u], acc);
    }
    store_out(out, out_off + i * out_stride_h + d, out_dtype, acc * w[ns]);
  }
  __syncthreads();
}

// The hand-off to the last CTA of a (b, kv head): every thread's partial
// writes are ordered before thread 0's fence and ticket increment by the CTA
// barrier; the CTA that draws the last ticket fences again before its threads
// read the other CTAs' partials. Returns true in that CTA (all threads).
__device__ __forceinline__ bool last_cta_ticket(uint32_t* ticket, int ns, int* s_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned t = atomicAdd(ticket, 1u);
    const int last = (t == unsigned(ns - 1)) ? 1 : 0;
    if (last) __threadfence();
    *s_flag = last;
  }
  __syncthreads();
  return *s_flag != 0;
}

// Writes the CTA's merged state for query head g of its kv head (or the final
// output when the split has a single chunk and the combine is fused), then, in
// fused mode, lets the last CTA of the kv head run the combine.
// `mrg_m`, `mrg_l` hold NW x G, `mrg_acc` NW x G x D floats.
template <int NW>
__device__ __forceinline__ void finish_cta(const DecodeArgs& a, int b, int h, int c,
                                           const float* mrg_m, const float* mrg_l,
                                           const float* mrg_acc, float* scratch) {
  const int tid = threadIdx.x;
  const int G = a.G, D = a.D;
  const int Hq = a.Hk * G;
  const bool direct = a.fuse && a.ns == 1;
  for (int i = tid; i < G * D; i += blockDim.x) {
    const int g = i / D, d = i - (i / D) * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w)
      if (mrg_l[w * G + g] > 0.f) M = fmaxf(M, mrg_m[w * G + g]);
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float lw = mrg_l[w * G + g];
      if (lw > 0.f) {
        const float e = exp2f(mrg_m[w * G + g] - M);
        L = fmaf(lw, e, L);
        acc = fmaf(mrg_acc[(w * G + g) * D + d], e, acc);
      }
    }
    const int hq = h * G + g;
    if (direct) {
      store_out(a.out, b * a.os_b + hq * a.os_h + d, a.out_dtype, acc / L);
    } else {
      const int64_t row = (int64_t(b) * Hq + hq) * a.ns + c;
      a.pacc[row * D + d] = acc;
      if (d == 0) {
        a.pm[row] = M;
        a.pl[row] = L;
      }
    }
  }
  if (direct || !a.fuse) return;
  // last CTA of this (b, kv head) to arrive merges all chunks: an atomic
  // ticket, no waiting
  __shared__ int s_last;
  if (!last_cta_ticket(a.tickets + (b * a.Hk + h), a.ns, &s_last)) return;
  const int64_t row = (int64_t(b) * Hq + h * G) * a.ns;
  combine_heads(a.pm + row, a.pl + row, a.pacc + row * D, G, a.ns, a.ns, D, scratch, a.out,
                b * a.os_b + (h * G) * a.os_h, a.os_h, a.out_dtype);
  if (tid == 0) a.tickets[b * a.Hk + h] = 0u;
}

template <typename T>
__device__ __forceinline__ constexpr bool is_i8() {
  return std::is_same_v<T, int8_t>;
}

// Warp sums of N values at once (N a power of two <= 16): at each of the
// first log2(N) butterfly levels a lane keeps half of its values and trades
// the other half, so 31 / 32 shuffles do the work of N full reductions. Lane l
// returns the sum of value l / (32 / N); the additions pair the same lanes in
// the same order as a per-value xor butterfly, so the sums are bitwise those.
template <int N>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[N], int lane) {
#pragma unroll
  for (int n = N, off = 16; n > 1; n >>= 1, off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = up ? v[i] : v[i + n / 2];
      const float keep = up ? v[i + n / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  float x = v[0];
#pragma unroll
  for (int off = 16 / N; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// 2^x on the special-function unit (ex2.approx.ftz: 2^-inf = +0)
__device__ __forceinline__ float fast_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int VEC, int G, typename KT, typename VT>
__global__ void __launch_bounds__(kGenericWarps * 32)
    decode_generic_kernel(DecodeArgs a, Basis basis) {
  constexpr int NW = kGenericWarps;
  __shared__ float A_sm[kMaxR * kMaxS];  // A[t][j] = M[j][t], row t stride S
  __shared__ float s_sm[NW][kMaxS * G];
  __shared__ float p_sm[NW][kMaxR * G];
  __shared__ float w_sm[NW][kMaxS * G];
  __shared__ float mx_sm[NW][G], ps_sm[NW][G];  // per-head block maxima and sums
  __shared__ float mrg_m[NW * G], mrg_l[NW * G];
  extern __shared__ float dyn[];  // NW * G * D merge buffer, reused for combine weights

  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int R = a.R, S = a.S, D = a.D;
  int RS = 1;  // softmax segment: the power of two >= R
  while (RS < R) RS <<= 1;
  const int HP = 32 / RS;  // heads per logits pass
  const int tok = lane & (RS - 1), hp = lane / RS;
  for (int i = tid; i < R * S; i += blockDim.x) {
    const int t = i / S, j = i - (i / S) * S;
    A_sm[i] = basis.m[j][t];
  }
  float qv[G][VEC];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int v = 0; v < VEC; ++v)
      qv[g][v] = load_any(a.q, b * a.qs_b + (h * G + g) * a.qs_h + lane * VEC + v, a.q_dtype) *
                 a.qscale;
  float m[G], l[G], acc[G][VEC];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[g][v] = 0.f;
  }
  __syncthreads();

  const int64_t n0 = int64_t(c) * a.chunk;
  const int64_t n1 = min(n0 + a.chunk, a.nb);
  const KT* kbase = static_cast<const KT*>(a.kc) + b * a.kcs_b + h * a.kcs_h + lane * VEC;
  const VT* vbase = static_cast<const VT*>(a.vc) + b * a.vcs_b + h * a.vcs_h + lane * VEC;
  const float* ksb = a.ks ? a.ks + b * a.kss_b + h * a.kss_h : nullptr;
  const float* vsb = a.vs ? a.vs + b * a.vss_b + h * a.vss_h : nullptr;
  // a block of at most kPre rows (and lanes of at most 4 channels) has all its
  // K and V rows and scales requested at once: one memory round trip per block
  constexpr int kPre = 4;
  const bool pre = VEC <= 4 && S <= kPre;
  for (int64_t n = n0 + warp; n < n1; n += NW) {
    const KT* krow = kbase + n * S * D;
    const VT* vrow = vbase + n * S * D;
    float kb[kPre][VEC], vb[kPre][VEC], kscb[kPre];
    float vs_mine = 1.f;  // V scale of row lane / G (the lane's first w_j)
    if (pre) {
#pragma unroll
      for (int j = 0; j < kPre; ++j) {
        if (j < S) {
          load_vec<KT, VEC>(krow + int64_t(j) * D, kb[j]);
          load_vec<VT, VEC>(vrow + int64_t(j) * D, vb[j]);
          kscb[j] = 1.f;
          if constexpr (is_i8<KT>()) kscb[j] = __ldg(ksb + n * S + j);
        }
      }
      if constexpr (is_i8<VT>()) {
        if (lane < S * G) vs_mine = __ldg(vsb + n * S + lane / G);
      }
    }
    // s_j = scale_kj * (C_k[j] . q) for every kept frequency j
    auto k_row = [&](int j, const float (&kf)[VEC], float ksc) {
      float part[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float x = 0.f;
#pragma unroll
        for (int v = 0; v < VEC; ++v) x = fmaf(kf[v], qv[g][v], x);
        part[g] = x;
      }
      const float tot = warp_reduce_scatter<G>(part, lane);  // head lane / (32 / G)
      if ((lane & (32 / G - 1)) == 0) s_sm[warp][j * G + lane / (32 / G)] = tot * ksc;
    };
    if (pre) {
#pragma unroll
      for (int j = 0; j < kPre; ++j)
        if (j < S) k_row(j, kb[j], kscb[j]);
    } else {
      for (int j = 0; j < S; ++j) {
        float kf[VEC];
        load_vec<KT, VEC>(krow + int64_t(j) * D, kf);
        float ksc = 1.f;
        if constexpr (is_i8<KT>()) ksc = __ldg(ksb + n * S + j);
        k_row(j, kf, ksc);
      }
    }
    __syncwarp();
    // logits: lane = (token t, head slot hp) in segments of RS >= R lanes, HP
    // heads per pass; per-segment max and sum, then every lane takes the new
    // maxima and sums of all heads from shared memory
    for (int g0 = 0; g0 < G; g0 += HP) {
      const int g = g0 + hp;
      const bool live = tok < R && g < G;
      float lg = -INFINITY;
      if (live) {
        lg = 0.f;
        for (int j = 0; j < S; ++j) lg = fmaf(A_sm[tok * S + j], s_sm[warp][j * G + g], lg);
      }
      float mo = m[0];
#pragma unroll
      for (int gg = 1; gg < G; ++gg) mo = (gg == g) ? m[gg] : mo;
      float mx = lg;
      for (int off = RS / 2; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float mn = fmaxf(mo, mx);
      const float p = live ? fast_ex2(lg - mn) : 0.f;
      float ps = p;
      for (int off = RS / 2; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      if (live) p_sm[warp][tok * G + g] = p;
      if (tok == 0 && g < G) {
        mx_sm[warp][g] = mn;
        ps_sm[warp][g] = ps;
      }
    }
    __syncwarp();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mn = mx_sm[warp][g];
      const float alpha = fast_ex2(m[g] - mn);
      l[g] = fmaf(l[g], alpha, ps_sm[warp][g]);
      m[g] = mn;
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[g][v] *= alpha;
    }
    __syncwarp();
    // w_j = scale_vj * sum_t p_t A[t][j]
    for (int i = lane; i < S * G; i += 32) {
      const int j = i / G, g = i - (i / G) * G;
      float x = 0.f;
      for (int t = 0; t < R; ++t) x = fmaf(p_sm[warp][t * G + g], A_sm[t * S + j], x);
      if constexpr (is_i8<VT>()) x *= (pre && i == lane) ? vs_mine : __ldg(vsb + n * S + j);
      w_sm[warp][i] = x;
    }
    __syncwarp();
    // acc += w C_v
    auto v_row = [&](int j, const float (&vf)[VEC]) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float wg = w_sm[warp][j * G + g];
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[g][v] = fmaf(wg, vf[v], acc[g][v]);
      }
    };
    if (pre) {
#pragma unroll
      for (int j = 0; j < kPre; ++j)
        if (j < S) v_row(j, vb[j]);
    } else {
      for (int j = 0; j < S; ++j) {
        float vf[VEC];
        load_vec<VT, VEC>(vrow + int64_t(j) * D, vf);
        v_row(j, vf);
      }
    }
    __syncwarp();
  }

  // raw tail tokens: the last chunk folds them into the same softmax
  if (c == a.ns - 1) {
    for (int i = warp; i < a.nr; i += NW) {
      float kf[VEC], vf[VEC];
      const int64_t koff = b * a.kts_b + h * a.kts_h + int64_t(i) * D + lane * VEC;
      const int64_t voff = b * a.vts_b + h * a.vts_h + int64_t(i) * D + lane * VEC;
#pragma unroll
      for (int v = 0; v < VEC; ++v) {
        kf[v] = load_any(a.kt, koff + v, a.t_dtype);
        vf[v] = load_any(a.vt, voff + v, a.t_dtype);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float part = 0.f;
#pragma unroll
        for (int v = 0; v < VEC; ++v) part = fmaf(kf[v], qv[g][v], part);
        const float lg = warp_sum(part);
        const float mn = fmaxf(m[g], lg);
        const float p = exp2f(lg - mn);
        const float alpha = exp2f(m[g] - mn);
        l[g] = fmaf(l[g], alpha, p);
        m[g] = mn;
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[g][v] = fmaf(acc[g][v], alpha, p * vf[v]);
      }
    }
  }

  // merge the NW warp states of this CTA
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      mrg_m[warp * G + g] = m[g];
      mrg_l[warp * G + g] = l[g];
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int v = 0; v < VEC; ++v) dyn[(warp * G + g) * D + lane * VEC + v] = acc[g][v];
  __syncthreads();
  finish_cta<NW>(a, b, h, c, mrg_m, mrg_l, dyn, dyn + NW * G * D);
}

// Shared memory (bytes) the generic kernel needs beyond its static arrays:
// the warp-merge buffer, followed by the combine weights.
inline size_t generic_dyn_smem(int G, int D, int ns) {
  return size_t(kGenericWarps * G * D + G * (ns + 1)) * sizeof(float);
}

// Launchers, one explicit instantiation per (K, V) coefficient type pair.
template <typename KT, typename VT>
int launch_decode_generic(const DecodeArgs& a, const Basis& basis, cudaStream_t stream);

// Tensor-core kernel for int8 K and V archives (fc_decode_tc.cu).
bool decode_tc_eligible(const fc_archive* ka, const fc_archive* va, int G);
int tc_tiles_per_head(int64_t nb, int S);
int launch_decode_tc(const DecodeArgs& d, const fc_archive* ka, const fc_archive* va, const Basis& basis,
                     cudaStream_t stream);
// The problems d[0..n) (same G, S, R; each tensor-core eligible) in one launch.
int launch_decode_tc_layers(int n, const DecodeArgs* d, const fc_archive* const* ka, const fc_archive* const* va,
                            const Basis& basis, cudaStream_t stream);

// Combine kernel for fc_combine: one CTA per (b, q head).
struct CombineArgs {
  const float* pm;
  const float* pl;
  const float* pacc;
  int Hq, D, ns;
  void* out;
  int out_dtype;
  int64_t os_b, os_h;
};

}  // namespace fc
