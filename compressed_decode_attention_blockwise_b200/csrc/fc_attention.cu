// Entry points of coefficient-domain decode attention: planning, argument
// validation, kernel selection, and the stand-alone combine.
#include <cmath>
#include <mutex>

#include "fc_decode.cuh"

namespace fc {
namespace {

// Split count. The tensor-core kernel runs one CTA per SM (its two rings of
// 128-row tiles fill the shared memory): split each kv head into tile-aligned
// chunks so that all chunks of all kv heads fit in one wave (rounded down:
// the SMs left over let the next launch on the stream start early). The
// portable kernel fits four CTAs per SM (registers) and aims at one wave of
// them, with chunks of at least 16 blocks.
// Results do not depend on the split beyond rounding.
int plan_splits(int64_t nb, int64_t B, int64_t Hk, int S, int D) {
  if (nb <= 0) return 1;
  const int64_t units = B * Hk;
  const bool tiles = D == 128 && S >= 1 && 32 % S == 0;
  int64_t ns;
  if (tiles) {
    ns = int64_t(sm_count()) / units;
    const int64_t t = tc_tiles_per_head(nb, S);
    if (ns > t) ns = t;
  } else {
    // rounded down: a partial second wave of CTAs would double the time
    ns = int64_t(sm_count()) * 4 / units;
    const int64_t by_len = nb / 16 > 0 ? nb / 16 : 1;
    if (ns > by_len) ns = by_len;
  }
  if (ns > kMaxSplits) ns = kMaxSplits;
  if (ns < 1) ns = 1;
  return int(ns);
}

bool supported_G(int64_t G) { return G == 1 || G == 2 || G == 4 || G == 8 || G == 16; }

__global__ void __launch_bounds__(128) combine_kernel(CombineArgs a) {
  extern __shared__ float wts[];  // ns + 1
  const int hq = blockIdx.x, b = blockIdx.y;
  const int64_t row = (int64_t(b) * a.Hq + hq) * a.ns;
  combine_heads(a.pm + row, a.pl + row, a.pacc + row * a.D, 1, a.ns, a.ns, a.D, wts, a.out,
                b * a.os_b + hq * a.os_h, a.os_h, a.out_dtype);
}

int check_io(const void* p, int dtype, const int64_t* strides) {
  if (!p || !strides) return FC_ERR_INVALID;
  if (dtype != FC_DTYPE_F32 && dtype != FC_DTYPE_BF16) return FC_ERR_INVALID;
  if (strides[3] != 1 || strides[0] < 0 || strides[1] < 0) return FC_ERR_INVALID;
  return FC_OK;
}

}  // namespace
}  // namespace fc

using namespace fc;

extern "C" int fc_decode_plan(const fc_archive* ka, const fc_tail* kt, int64_t Hq,
                              int32_t* num_splits_out) {
  (void)kt;
  if (!num_splits_out) return FC_ERR_INVALID;
  const int st = check_archive(ka);
  if (st != FC_OK) return st;
  if (Hq < 1 || Hq % ka->H) return FC_ERR_INVALID;
  *num_splits_out = plan_splits(ka->n_blocks, ka->B, ka->H, ka->S, int(ka->D));
  return FC_OK;
}

extern "C" int fc_decode_kernel(const fc_archive* ka, const fc_archive* va, int64_t Hq, int32_t flags,
                                int32_t* kind_out) {
  if (!kind_out || !va) return FC_ERR_INVALID;
  int st = check_archive(ka);
  if (st != FC_OK) return st;
  st = check_archive(va);
  if (st != FC_OK) return st;
  if (Hq < 1 || Hq % ka->H) return FC_ERR_INVALID;
  *kind_out = (!(flags & FC_DECODE_PORTABLE) && decode_tc_eligible(ka, va, int(Hq / ka->H)))
                  ? FC_KERNEL_TENSOR_CORE
                  : FC_KERNEL_CUDA_CORE;
  return FC_OK;
}

namespace fc {
namespace {

// Validation and argument set-up shared by fc_decode_attention and
// fc_decode_step. `extra_token`: a new token joins the softmax (the step), so
// an empty archive with an empty tail is valid.
int prepare_decode(const void* q, int32_t q_dtype, const int64_t* q_strides, int64_t Hq,
                   const fc_archive* ka, const fc_archive* va, const fc_tail* kt, const fc_tail* vt,
                   float softmax_scale, int32_t num_splits, int32_t flags, void* workspace,
                   size_t workspace_bytes, void* out, int32_t out_dtype, const int64_t* out_strides,
                   bool extra_token, DecodeArgs* ap) {
  int st = check_archive(ka);
  if (st != FC_OK) return st;
  st = check_archive(va);
  if (st != FC_OK) return st;
  if (ka->B != va->B || ka->H != va->H || ka->R != va->R || ka->S != va->S || ka->D != va->D ||
      ka->n_blocks != va->n_blocks)
    return FC_ERR_INVALID;
  st = check_io(q, q_dtype, q_strides);
  if (st != FC_OK) return st;
  st = check_io(out, out_dtype, out_strides);
  if (st != FC_OK) return st;
  if (Hq < 1 || Hq % ka->H) return FC_ERR_INVALID;
  const int64_t G = Hq / ka->H;
  if (!supported_G(G)) return FC_ERR_UNSUPPORTED;
  if (G * (ka->D / 32) > 64) return FC_ERR_UNSUPPORTED;
  int nr = 0;
  int t_dtype = FC_DTYPE_BF16;
  if (kt || vt) {
    if (!kt || !vt) return FC_ERR_INVALID;
    st = check_tail(kt, ka, true);
    if (st != FC_OK) return st;
    st = check_tail(vt, va, true);
    if (st != FC_OK) return st;
    if (kt->len != vt->len || kt->dtype != vt->dtype) return FC_ERR_INVALID;
    nr = kt->len;
    t_dtype = kt->dtype;
  }
  if (ka->n_blocks == 0 && nr == 0 && !extra_token) return FC_ERR_INVALID;
  int ns = num_splits;
  if (ns == 0) ns = plan_splits(ka->n_blocks, ka->B, ka->H, ka->S, int(ka->D));
  if (ns < 1 || ns > kMaxSplits) return FC_ERR_INVALID;
  if (flags & ~(FC_DECODE_FUSE_COMBINE | FC_DECODE_PORTABLE | FC_DECODE_OVERLAP | FC_DECODE_Q_FINAL |
                FC_DECODE_TEST_TIMEOUT))
    return FC_ERR_INVALID;
  const bool fuse_combine = (flags & FC_DECODE_FUSE_COMBINE) != 0;
  if (ka->B > 65535 || ka->H > 65535) return FC_ERR_UNSUPPORTED;
  const bool need_ws = !(fuse_combine && ns == 1);
  if (flags & FC_DECODE_TEST_TIMEOUT) {
    if (!need_ws) return FC_ERR_INVALID;  // no status word to record the error in
    if ((flags & FC_DECODE_PORTABLE) || !decode_tc_eligible(ka, va, int(G))) return FC_ERR_UNSUPPORTED;
  }
  const WorkspaceLayout wl = workspace_layout(ka->B, Hq, ka->D, ns);
  if (need_ws) {
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
        workspace_bytes < wl.total)
      return FC_ERR_INVALID;
  }
  DecodeArgs a = {};
  a.q = q;
  a.q_dtype = q_dtype;
  a.qs_b = q_strides[0];
  a.qs_h = q_strides[1];
  a.kc = ka->coeffs;
  a.ks = ka->scales;
  a.kcs_b = ka->coeff_stride_b;
  a.kcs_h = ka->coeff_stride_h;
  a.kss_b = ka->scale_stride_b;
  a.kss_h = ka->scale_stride_h;
  a.vc = va->coeffs;
  a.vs = va->scales;
  a.vcs_b = va->coeff_stride_b;
  a.vcs_h = va->coeff_stride_h;
  a.vss_b = va->scale_stride_b;
  a.vss_h = va->scale_stride_h;
  a.kt = kt ? kt->data : nullptr;
  a.vt = vt ? vt->data : nullptr;
  a.t_dtype = t_dtype;
  a.kts_b = kt ? kt->stride_b : 0;
  a.kts_h = kt ? kt->stride_h : 0;
  a.vts_b = vt ? vt->stride_b : 0;
  a.vts_h = vt ? vt->stride_h : 0;
  a.nr = nr;
  a.B = int(ka->B);
  a.Hk = int(ka->H);
  a.G = int(G);
  a.R = ka->R;
  a.S = ka->S;
  a.D = int(ka->D);
  a.nb = ka->n_blocks;
  a.ns = ns;
  a.chunk = ka->n_blocks > 0 ? (ka->n_blocks + ns - 1) / ns : 0;
  // the uneven automatic split needs the fused combine (fc_combine merges
  // ns slots for every head)
  a.auto_split = (num_splits == 0 && fuse_combine) ? 1 : 0;
  a.bal_q = ns;
  a.bal_rem = 0;
  const float sigma = softmax_scale > 0.f ? softmax_scale : float(1.0 / std::sqrt(double(ka->D)));
  a.qscale = float(double(sigma) * 1.4426950408889634);  // log2(e)
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.status = need_ws ? reinterpret_cast<uint32_t*>(ws + wl.status) : nullptr;
  a.tickets = need_ws ? reinterpret_cast<uint32_t*>(ws + wl.tickets) : nullptr;
  a.pm = need_ws ? reinterpret_cast<float*>(ws + wl.m) : nullptr;
  a.pl = need_ws ? reinterpret_cast<float*>(ws + wl.l) : nullptr;
  a.pacc = need_ws ? reinterpret_cast<float*>(ws + wl.acc) : nullptr;
  a.fuse = fuse_combine ? 1 : 0;
  a.overlap = (flags & FC_DECODE_OVERLAP) ? 1 : 0;
  a.q_final = (a.overlap && (flags & FC_DECODE_Q_FINAL)) ? 1 : 0;
  a.test_stall = (flags & FC_DECODE_TEST_TIMEOUT) ? 1 : 0;
  a.out = out;
  a.out_dtype = out_dtype;
  a.os_b = out_strides[0];
  a.os_h = out_strides[1];
  a.step = 0;
  *ap = a;
  return FC_OK;
}

int launch_prepared(const DecodeArgs& a, const fc_archive* ka, const fc_archive* va, int32_t flags,
                    cudaStream_t stream) {
  Basis basis;
  make_basis(ka->codec, ka->R, ka->S, &basis);
  if (!(flags & FC_DECODE_PORTABLE) && decode_tc_eligible(ka, va, a.G))
    return launch_decode_tc(a, ka, va, basis, stream);
  const int kd = ka->coeff_dtype, vd = va->coeff_dtype;
  if (kd == FC_DTYPE_I8 && vd == FC_DTYPE_I8) return launch_decode_generic<int8_t, int8_t>(a, basis, stream);
  if (kd == FC_DTYPE_I8 && vd == FC_DTYPE_BF16)
    return launch_decode_generic<int8_t, __nv_bfloat16>(a, basis, stream);
  if (kd == FC_DTYPE_I8 && vd == FC_DTYPE_F32) return launch_decode_generic<int8_t, float>(a, basis, stream);
  if (kd == FC_DTYPE_BF16 && vd == FC_DTYPE_BF16)
    return launch_decode_generic<__nv_bfloat16, __nv_bfloat16>(a, basis, stream);
  if (kd == FC_DTYPE_F32 && vd == FC_DTYPE_F32) return launch_decode_generic<float, float>(a, basis, stream);
  return FC_ERR_UNSUPPORTED;
}

StreamOut out_of(const fc_archive* a) {
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

extern "C" int fc_decode_attention(const void* q, int32_t q_dtype, const int64_t* q_strides,
                                   int64_t Hq, const fc_archive* ka, const fc_archive* va,
                                   const fc_tail* kt, const fc_tail* vt, float softmax_scale,
                                   int32_t num_splits, int32_t flags, void* workspace,
                                   size_t workspace_bytes, void* out, int32_t out_dtype,
                                   const int64_t* out_strides, fc_stream stream) {
  DecodeArgs a;
  const int st = prepare_decode(q, q_dtype, q_strides, Hq, ka, va, kt, vt, softmax_scale, num_splits, flags,
                                workspace, workspace_bytes, out, out_dtype, out_strides, false, &a);
  if (st != FC_OK) return st;
  return launch_prepared(a, ka, va, flags, stream);
}

namespace fc {
namespace {

// Argument set-up of one fused decode step (fc_decode_step): *fused tells
// whether the tensor-core kernel serves it in one launch (then *ap holds the
// step fields and *complete whether the token completes a block); otherwise
// the caller issues fc_append_step + fc_decode_attention.
int prepare_step(const void* q, int32_t q_dtype, const int64_t* q_strides, int64_t Hq, const void* k_new,
                 const void* v_new, int32_t new_dtype, const int64_t* k_strides, const int64_t* v_strides,
                 const fc_archive* ka, const fc_archive* va, const fc_tail* kt, const fc_tail* vt,
                 float softmax_scale, int32_t num_splits, int32_t flags, void* workspace,
                 size_t workspace_bytes, void* out, int32_t out_dtype, const int64_t* out_strides,
                 DecodeArgs* ap, bool* fused, bool* complete) {
  if (!k_new || !v_new || !k_strides || !v_strides || !kt || !vt || !kt->data || !vt->data)
    return FC_ERR_INVALID;
  if (flags & FC_DECODE_TEST_TIMEOUT) return FC_ERR_INVALID;  // fc_decode_attention only
  DecodeArgs a;
  int st = prepare_decode(q, q_dtype, q_strides, Hq, ka, va, kt, vt, softmax_scale, num_splits, flags,
                          workspace, workspace_bytes, out, out_dtype, out_strides, true, &a);
  if (st != FC_OK) return st;
  *fused = !(flags & FC_DECODE_PORTABLE) && decode_tc_eligible(ka, va, a.G) && new_dtype == kt->dtype &&
           k_strides[3] == 1 && v_strides[3] == 1 && aligned16(k_new) && aligned16(v_new) &&
           k_strides[0] >= 0 && k_strides[1] >= 0 && v_strides[0] >= 0 && v_strides[1] >= 0;
  if (!*fused) return FC_OK;
  const int esz = dtype_size(new_dtype);
  if ((k_strides[0] * esz) % 16 || (k_strides[1] * esz) % 16 || (v_strides[0] * esz) % 16 ||
      (v_strides[1] * esz) % 16)
    return FC_ERR_INVALID;
  *complete = kt->len + 1 == ka->R;
  if (*complete && (ka->n_blocks >= ka->capacity || va->n_blocks >= va->capacity)) return FC_ERR_CAPACITY;
  a.step = *complete ? 2 : 1;
  a.kn = k_new;
  a.vn = v_new;
  a.kns_b = k_strides[0];
  a.kns_h = k_strides[1];
  a.vns_b = v_strides[0];
  a.vns_h = v_strides[1];
  a.kout = out_of(ka);
  a.vout = out_of(va);
  a.new_slot = ka->n_blocks;
  *ap = a;
  return FC_OK;
}

// host descriptors after a step: the token joined the tail or completed a block
void advance_step(fc_archive* ka, fc_archive* va, fc_tail* kt, fc_tail* vt, bool complete) {
  if (complete) {
    ka->n_blocks += 1;
    va->n_blocks += 1;
    kt->len = 0;
    vt->len = 0;
  } else {
    kt->len += 1;
    vt->len += 1;
  }
}

}  // namespace
}  // namespace fc

extern "C" int fc_decode_step(const void* q, int32_t q_dtype, const int64_t* q_strides, int64_t Hq,
                              const void* k_new, const void* v_new, int32_t new_dtype,
                              const int64_t* k_strides, const int64_t* v_strides, fc_archive* ka,
                              fc_archive* va, fc_tail* kt, fc_tail* vt, float softmax_scale,
                              int32_t num_splits, int32_t flags, void* workspace,
                              size_t workspace_bytes, void* out, int32_t out_dtype,
                              const int64_t* out_strides, fc_stream stream) {
  DecodeArgs a;
  bool fused = false, complete = false;
  int st = prepare_step(q, q_dtype, q_strides, Hq, k_new, v_new, new_dtype, k_strides, v_strides, ka, va, kt, vt,
                        softmax_scale, num_splits, flags, workspace, workspace_bytes, out, out_dtype,
                        out_strides, &a, &fused, &complete);
  if (st != FC_OK) return st;
  if (!fused) {
    // two launches: the append, then the attention over the updated stream
    st = fc_append_step(k_new, v_new, new_dtype, k_strides, v_strides, ka, va, kt, vt, stream);
    if (st != FC_OK) return st;
    return fc_decode_attention(q, q_dtype, q_strides, Hq, ka, va, kt, vt, softmax_scale, num_splits, flags,
                               workspace, workspace_bytes, out, out_dtype, out_strides, stream);
  }
  st = launch_prepared(a, ka, va, flags, stream);
  if (st != FC_OK) return st;
  advance_step(ka, va, kt, vt, complete);
  return FC_OK;
}

namespace fc {
namespace {

struct StagingLayout {
  size_t k, v, q, out, total;
};

StagingLayout staging_layout(int64_t B, int64_t H, int64_t Hq, int64_t D, int io_dtype, int out_dtype) {
  StagingLayout s;
  const size_t tok = size_t(B) * size_t(H) * size_t(D) * size_t(dtype_size(io_dtype));
  const size_t qb = size_t(B) * size_t(Hq) * size_t(D) * size_t(dtype_size(io_dtype));
  s.k = 0;
  s.v = pad256(tok);
  s.q = s.v + pad256(tok);
  s.out = s.q + pad256(qb);
  s.total = s.out + pad256(size_t(B) * size_t(Hq) * size_t(D) * size_t(dtype_size(out_dtype)));
  return s;
}

}  // namespace
}  // namespace fc

extern "C" size_t fc_decode_step_staging_bytes(int64_t B, int64_t H, int64_t Hq, int64_t D, int32_t io_dtype,
                                               int32_t out_dtype) {
  if (B < 1 || H < 1 || Hq < 1 || D < 1) return 0;
  if ((io_dtype != FC_DTYPE_BF16 && io_dtype != FC_DTYPE_F32) ||
      (out_dtype != FC_DTYPE_BF16 && out_dtype != FC_DTYPE_F32))
    return 0;
  return staging_layout(B, H, Hq, D, io_dtype, out_dtype).total;
}

extern "C" int fc_decode_step_host(const void* in_host, void* out_host, void* staging, size_t staging_bytes,
                                   int32_t io_dtype, int32_t out_dtype, int64_t Hq, fc_archive* ka,
                                   fc_archive* va, fc_tail* kt, fc_tail* vt, float softmax_scale,
                                   int32_t num_splits, int32_t flags, void* workspace, size_t workspace_bytes,
                                   fc_stream stream) {
  if (!in_host || !out_host || !staging || (reinterpret_cast<uintptr_t>(staging) & 255u)) return FC_ERR_INVALID;
  int st = check_archive(ka);
  if (st != FC_OK) return st;
  const size_t need = fc_decode_step_staging_bytes(ka->B, ka->H, Hq, ka->D, io_dtype, out_dtype);
  if (need == 0 || staging_bytes < need) return FC_ERR_INVALID;
  const StagingLayout L = staging_layout(ka->B, ka->H, Hq, ka->D, io_dtype, out_dtype);
  uint8_t* sg = static_cast<uint8_t*>(staging);
  const size_t esz = size_t(dtype_size(io_dtype));
  const size_t tok = size_t(ka->B * ka->H * ka->D) * esz;
  const size_t qb = size_t(ka->B * Hq * ka->D) * esz;
  const int64_t tok_s[4] = {ka->H * ka->D, ka->D, ka->D, 1};
  const int64_t q_s[4] = {Hq * ka->D, ka->D, ka->D, 1};
  {
    // every argument is checked before any copy or kernel is queued
    DecodeArgs chk;
    bool fused = false, complete = false;
    st = prepare_step(sg + L.q, io_dtype, q_s, Hq, sg + L.k, sg + L.v, io_dtype, tok_s, tok_s, ka, va, kt, vt,
                      softmax_scale, num_splits, flags, workspace, workspace_bytes, sg + L.out, out_dtype, q_s,
                      &chk, &fused, &complete);
    if (st != FC_OK) return st;
  }
  // pinned host memory that the device can address (mapped, as every pinned
  // allocation is under unified addressing): the kernels read the inputs and
  // write the output there directly, and the copies happen inside them
  cudaPointerAttributes pin{}, pout{};
  if (cudaPointerGetAttributes(&pin, in_host) == cudaSuccess &&
      cudaPointerGetAttributes(&pout, out_host) == cudaSuccess && pin.type == cudaMemoryTypeHost &&
      pout.type == cudaMemoryTypeHost && pin.devicePointer && pout.devicePointer) {
    const uint8_t* din = static_cast<const uint8_t*>(pin.devicePointer);
    return fc_decode_step(din + 2 * tok, io_dtype, q_s, Hq, din, din + tok, io_dtype, tok_s, tok_s, ka, va, kt, vt,
                          softmax_scale, num_splits, flags, workspace, workspace_bytes, pout.devicePointer,
                          out_dtype, q_s, stream);
  }
  (void)cudaGetLastError();  // pageable memory: an unregistered pointer is not an error here
  // the host block is [k_new | v_new | q], each contiguous (B, heads, 1, D);
  // one copy when the staging offsets are contiguous too, else three
  const uint8_t* in = static_cast<const uint8_t*>(in_host);
  cudaError_t e = cudaSuccess;
  if (L.v == tok && L.q == 2 * tok) {
    e = cudaMemcpyAsync(sg, in, 2 * tok + qb, cudaMemcpyHostToDevice, stream);
  } else {
    e = cudaMemcpyAsync(sg + L.k, in, tok, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(sg + L.v, in + tok, tok, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaMemcpyAsync(sg + L.q, in + 2 * tok, qb, cudaMemcpyHostToDevice, stream);
  }
  if (e != cudaSuccess) return FC_ERR_CUDA;
  st = fc_decode_step(sg + L.q, io_dtype, q_s, Hq, sg + L.k, sg + L.v, io_dtype, tok_s, tok_s, ka, va, kt, vt,
                      softmax_scale, num_splits, flags, workspace, workspace_bytes, sg + L.out, out_dtype, q_s,
                      stream);
  if (st != FC_OK) return st;
  const size_t ob = size_t(ka->B * Hq * ka->D) * size_t(dtype_size(out_dtype));
  return cuda_status(cudaMemcpyAsync(out_host, sg + L.out, ob, cudaMemcpyDeviceToHost, stream));
}

extern "C" int fc_decode_step_layers(int32_t n_layers, fc_layer_step* layers, int32_t q_dtype,
                                     int32_t new_dtype, int32_t out_dtype, int64_t Hq, float softmax_scale,
                                     int32_t num_splits, int32_t flags, fc_stream stream) {
  if (n_layers < 1 || n_layers > FC_MAX_LAYERS || !layers) return FC_ERR_INVALID;
  if (flags & FC_DECODE_PORTABLE) return FC_ERR_INVALID;
  DecodeArgs args[FC_MAX_LAYERS];
  const fc_archive* kas[FC_MAX_LAYERS];
  const fc_archive* vas[FC_MAX_LAYERS];
  bool complete[FC_MAX_LAYERS];
  for (int i = 0; i < n_layers; ++i) {
    fc_layer_step& L = layers[i];
    bool fused = false;
    const int st = prepare_step(L.q, q_dtype, L.q_strides, Hq, L.k_new, L.v_new, new_dtype, L.k_strides,
                                L.v_strides, L.ka, L.va, L.kt, L.vt, softmax_scale, num_splits, flags,
                                L.workspace, L.workspace_bytes, L.out, out_dtype, L.out_strides, &args[i],
                                &fused, &complete[i]);
    if (st != FC_OK) return st;
    if (!fused) return FC_ERR_UNSUPPORTED;
    if (args[i].G != args[0].G || args[i].S != args[0].S || args[i].R != args[0].R ||
        args[i].D != args[0].D)
      return FC_ERR_UNSUPPORTED;
    for (int j = 0; j < i; ++j)  // one launch writes every layer's streams
      if (layers[j].ka == L.ka || layers[j].va == L.va || layers[j].kt == L.kt || layers[j].vt == L.vt ||
          layers[j].workspace == L.workspace)
        return FC_ERR_INVALID;
    kas[i] = L.ka;
    vas[i] = L.va;
  }
  Basis basis;
  make_basis(FC_CODEC_DCT, args[0].R, args[0].S, &basis);
  const int st = launch_decode_tc_layers(n_layers, args, kas, vas, basis, stream);
  if (st != FC_OK) return st;
  for (int i = 0; i < n_layers; ++i)
    advance_step(layers[i].ka, layers[i].va, layers[i].kt, layers[i].vt, complete[i]);
  return FC_OK;
}

extern "C" int fc_combine(const void* workspace, size_t workspace_bytes, int64_t B, int64_t Hq,
                          int64_t D, int32_t num_splits, void* out, int32_t out_dtype,
                          const int64_t* out_strides, fc_stream stream) {
  if (B < 1 || Hq < 1 || num_splits < 1 || num_splits > kMaxSplits) return FC_ERR_INVALID;
  if (D != 32 && D != 64 && D != 128 && D != 256) return FC_ERR_UNSUPPORTED;
  int st = check_io(out, out_dtype, out_strides);
  if (st != FC_OK) return st;
  const WorkspaceLayout wl = workspace_layout(B, Hq, D, num_splits);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < wl.total)
    return FC_ERR_INVALID;
  if (B > 65535 || Hq > 0x7fffffff) return FC_ERR_UNSUPPORTED;
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  CombineArgs a;
  a.pm = reinterpret_cast<const float*>(ws + wl.m);
  a.pl = reinterpret_cast<const float*>(ws + wl.l);
  a.pacc = reinterpret_cast<const float*>(ws + wl.acc);
  a.Hq = int(Hq);
  a.D = int(D);
  a.ns = num_splits;
  a.out = out;
  a.out_dtype = out_dtype;
  a.os_b = out_strides[0];
  a.os_h = out_strides[1];
  const size_t smem = size_t(num_splits + 1) * sizeof(float);
  combine_kernel<<<dim3(unsigned(Hq), unsigned(B)), 128, smem, stream>>>(a);
  return cuda_status(cudaGetLastError());
}

// ----------------------------------------------------------------------------
// Allocation-free decode attention: the scratch is a file-scope device array
// (FC_NOALLOC_SCRATCH_BYTES, held by every GPU that loads the library until the
// process exits). Host code cannot use the array's name as a device address,
// so its address is resolved with cudaGetSymbolAddress once per device, with
// that device current, on the first call made on the device.
namespace fc {
namespace {

__device__ __align__(256) uint8_t g_noalloc_scratch[FC_NOALLOC_SCRATCH_BYTES];

int noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FC_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return FC_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return FC_OK;
}

}  // namespace
}  // namespace fc

extern "C" int fc_decode_attention_noalloc(const void* q, int32_t q_dtype, const int64_t* q_strides,
                                           int64_t Hq, const fc_archive* ka, const fc_archive* va,
                                           const fc_tail* kt, const fc_tail* vt, float softmax_scale,
                                           int32_t num_splits, void* out, int32_t out_dtype,
                                           const int64_t* out_strides, fc_stream stream) {
  int st = check_archive(ka);
  if (st != FC_OK) return st;
  if (Hq < 1 || Hq % ka->H) return FC_ERR_INVALID;
  int ns = num_splits;
  if (ns == 0) ns = plan_splits(ka->n_blocks, ka->B, ka->H, ka->S, int(ka->D));
  if (ns < 1 || ns > kMaxSplits) return FC_ERR_INVALID;
  const WorkspaceLayout wl = workspace_layout(ka->B, Hq, ka->D, ns);
  if (wl.total > FC_NOALLOC_SCRATCH_BYTES) return FC_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != FC_OK) return st;
  // the tickets must start at zero (the array keeps whatever the previous
  // call left); the status word is not cleared here, so that an error a
  // kernel reported stays readable through fc_noalloc_status
  if (cudaMemsetAsync(static_cast<uint8_t*>(scratch) + wl.tickets, 0, wl.m - wl.tickets, stream) != cudaSuccess)
    return FC_ERR_CUDA;
  return fc_decode_attention(q, q_dtype, q_strides, Hq, ka, va, kt, vt, softmax_scale, num_splits,
                             FC_DECODE_FUSE_COMBINE, scratch, FC_NOALLOC_SCRATCH_BYTES, out, out_dtype,
                             out_strides, stream);
}

extern "C" int fc_noalloc_status(uint32_t* device_status, fc_stream stream) {
  if (!device_status) return FC_ERR_INVALID;
  void* scratch = nullptr;
  const int st = noalloc_scratch(&scratch);
  if (st != FC_OK) return st;
  return fc_workspace_status(scratch, FC_NOALLOC_SCRATCH_BYTES, device_status, stream);
}
