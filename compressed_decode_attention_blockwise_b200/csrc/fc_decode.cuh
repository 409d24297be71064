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
  int ns;
  int64_t chunk;
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
// pm[i * ns + c], pl[i * ns + c], pacc[(i * ns + c) * D + d]; its output goes to
// out[out_off + i * out_stride_h + d]. All threads of the CTA take part. Each
// thread first issues the loads of the partial accumulators of its first
// (head, channel) output (up to kPre of them) and only then do warps compute
// the per-head weights into shared scratch `wts` (NH * (ns + 1) floats), so
// both sets of L2 reads are in flight together; further outputs (more outputs
// than threads) and partials beyond kPre use batched loads. Partials written
// by other CTAs of the same launch are read through L2 (ld.cg).
__device__ __forceinline__ void combine_heads(const float* pm, const float* pl, const float* pacc, int NH,
                                              int ns, int D, float* wts, void* out, int64_t out_off,
                                              int64_t out_stride_h, int out_dtype) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int n_out = NH * D;
  constexpr int kPre = 24;
  // partials of my first output, requested before the weights are known
  const bool has_first = tid < n_out;
  const int fi = has_first ? tid / D : 0, fd = has_first ? tid - fi * D : 0;
  const float* fsrc = pacc + int64_t(fi) * ns * D + fd;
  float pre[kPre];
#pragma unroll
  for (int u = 0; u < kPre; ++u) pre[u] = (has_first && u < ns) ? __ldcg(fsrc + int64_t(u) * D) : 0.f;

  constexpr int kReg = 4;  // partial rows per lane kept in registers (ns <= 128)
  for (int i = warp; i < NH; i += nwarps) {
    const float* m = pm + int64_t(i) * ns;
    const float* l = pl + int64_t(i) * ns;
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
    const float* src = pacc + int64_t(i) * ns * D + d;
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
  combine_heads(a.pm + row, a.pl + row, a.pacc + row * D, G, a.ns, D, scratch, a.out,
                b * a.os_b + (h * G) * a.os_h, a.os_h, a.out_dtype);
  if (tid == 0) a.tickets[b * a.Hk + h] = 0u;
}

template <typename T>
__device__ __forceinline__ constexpr bool is_i8() {
  return std::is_same_v<T, int8_t>;
}

template <int VEC, int G, typename KT, typename VT>
__global__ void __launch_bounds__(kGenericWarps * 32)
    decode_generic_kernel(DecodeArgs a, Basis basis) {
  constexpr int NW = kGenericWarps;
  __shared__ float A_sm[kMaxR * kMaxS];  // A[t][j] = M[j][t], row t stride S
  __shared__ float s_sm[NW][kMaxS * G];
  __shared__ float p_sm[NW][kMaxR * G];
  __shared__ float w_sm[NW][kMaxS * G];
  __shared__ float mrg_m[NW * G], mrg_l[NW * G];
  extern __shared__ float dyn[];  // NW * G * D merge buffer, reused for combine weights

  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int R = a.R, S = a.S, D = a.D;
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
  for (int64_t n = n0 + warp; n < n1; n += NW) {
    // s_j = scale_kj * (C_k[j] . q) for every kept frequency j
    const KT* krow = kbase + n * S * D;
    for (int j = 0; j < S; ++j) {
      float kf[VEC];
      load_vec<KT, VEC>(krow + int64_t(j) * D, kf);
      float ksc = 1.f;
      if constexpr (is_i8<KT>()) ksc = __ldg(ksb + n * S + j);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float part = 0.f;
#pragma unroll
        for (int v = 0; v < VEC; ++v) part = fmaf(kf[v], qv[g][v], part);
        part = warp_sum(part);
        if (lane == 0) s_sm[warp][j * G + g] = part * ksc;
      }
    }
    __syncwarp();
    // logits for token t = lane, online-softmax update per query head
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float lg = -INFINITY;
      if (lane < R) {
        lg = 0.f;
        for (int j = 0; j < S; ++j) lg = fmaf(A_sm[lane * S + j], s_sm[warp][j * G + g], lg);
      }
      const float mn = fmaxf(m[g], warp_max(lg));
      const float p = lane < R ? exp2f(lg - mn) : 0.f;
      const float alpha = exp2f(m[g] - mn);
      l[g] = fmaf(l[g], alpha, warp_sum(p));
      m[g] = mn;
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[g][v] *= alpha;
      if (lane < R) p_sm[warp][lane * G + g] = p;
    }
    __syncwarp();
    // w_j = scale_vj * sum_t p_t A[t][j]
    for (int i = lane; i < S * G; i += 32) {
      const int j = i / G, g = i - (i / G) * G;
      float x = 0.f;
      for (int t = 0; t < R; ++t) x = fmaf(p_sm[warp][t * G + g], A_sm[t * S + j], x);
      if constexpr (is_i8<VT>()) x *= __ldg(vsb + n * S + j);
      w_sm[warp][i] = x;
    }
    __syncwarp();
    // acc += w C_v
    const VT* vrow = vbase + n * S * D;
    for (int j = 0; j < S; ++j) {
      float vf[VEC];
      load_vec<VT, VEC>(vrow + int64_t(j) * D, vf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float wg = w_sm[warp][j * G + g];
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[g][v] = fmaf(wg, vf[v], acc[g][v]);
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
