// api.cu -- the C ABI of libsla (declared in include/sla.h): argument
// validation, workspace layout and kernel launches.  No allocation, no
// synchronisation (except sla_read_device_status), no state between calls.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>

#include "sla_internal.h"
#include "sla_kernels.h"

namespace sla {

cudaError_t encode_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int N, int BH, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDPad), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDPad) * 2, static_cast<cuuint64_t>(N) * kDPad * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_map8(CUtensorMap* map, const void* base, int N, int BH, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDPad), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDPad), static_cast<cuuint64_t>(N) * kDPad};
  cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace sla

namespace {

thread_local char g_detail[256] = "";

}  // namespace

void sla::set_error_detail(const char* msg) { snprintf(g_detail, sizeof(g_detail), "%s", msg); }

using namespace sla;

namespace {

sla_status cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_detail, sizeof(g_detail), "%s: %s", where, cudaGetErrorString(e));
  return SLA_ERR_CUDA;
}

sla_status arg_fail(sla_status s, const char* what) {
  snprintf(g_detail, sizeof(g_detail), "%s", what);
  return s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sla_status check_shape(const sla_shape* s) {
  if (s == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "shape is null");
  if (s->B < 1 || s->H < 1 || s->N < 1 || s->d < 1 || s->bq < 1 || s->bkv < 1)
    return arg_fail(SLA_ERR_INVALID_ARG, "shape sizes must be positive");
  if (s->in_dtype != SLA_F32 && s->in_dtype != SLA_BF16) return arg_fail(SLA_ERR_INVALID_ARG, "in_dtype");
  if (s->d % 8 != 0 || s->d > kDPad) return arg_fail(SLA_ERR_UNSUPPORTED, "d must be a multiple of 8, <= 128");
  if (s->bq != 64 && s->bq != 128) return arg_fail(SLA_ERR_UNSUPPORTED, "bq must be 64 or 128");
  if (s->bkv != kBlockKV) return arg_fail(SLA_ERR_UNSUPPORTED, "bkv must be 64");
  if (s->N > kMaxN) return arg_fail(SLA_ERR_UNSUPPORTED, "N > 131072");
  if (static_cast<long long>(s->B) * s->H > 65535) return arg_fail(SLA_ERR_UNSUPPORTED, "B*H > 65535");
  return SLA_OK;
}

sla_status check_ws(const sla_shape* s, int mode, const void* ws, size_t ws_bytes) {
  if (ws == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "ws is null");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return arg_fail(SLA_ERR_ALIGNMENT, "ws must be 256-byte aligned");
  if (ws_bytes < ws_layout(*s, mode).total) return arg_fail(SLA_ERR_WORKSPACE, "ws smaller than sla_workspace_size");
  return SLA_OK;
}

sla_status check_qkv(const void* q, const void* k, const void* v) {
  if ((q == nullptr) || (k == nullptr) || (v == nullptr)) return arg_fail(SLA_ERR_INVALID_ARG, "Q, K or V is null");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return arg_fail(SLA_ERR_ALIGNMENT, "Q, K, V must be 16-byte aligned");
  return SLA_OK;
}

// attention kernel inputs shared by both modes
sla_status run_attention(const sla_shape* s, const void* q, const void* k, const void* v, int phi,
                         unsigned flags, const WsLayout& L, char* ws, cudaStream_t st, SparseArgs& a) {
  cudaError_t e;
  if (!(flags & SLA_FLAG_PREPARED)) {
    if ((e = launch_prepare(*s, k, v, phi, L, ws, st)) != cudaSuccess) return cuda_fail(e, "prepare");
  }
  if (L.need_hat) {
    if ((e = launch_qhat(*s, q, L, ws, st)) != cudaSuccess) return cuda_fail(e, "qhat");
  }
  a.fp8 = (flags & SLA_FLAG_INT8) ? 2 : ((flags & SLA_FLAG_FP8) ? 1 : 0);
  a.wait_ns = (flags & SLA_FLAG_WAIT_TEST) ? 0ull : kWaitLimitNs;
  a.nb128 = ceil_div(s->N, 128);
  if (a.fp8) {
    if ((e = launch_fp8_quant(*s, q, k, v, L, ws, st, a.fp8 == 2)) != cudaSuccess)
      return cuda_fail(e, "low-bit quantisation");
    a.sq = reinterpret_cast<const float*>(ws + L.sq);
    a.sk = reinterpret_cast<const float*>(ws + L.sk);
    a.vamax = reinterpret_cast<const float*>(ws + L.sv);
  }
  a.BH = s->B * s->H;
  a.N = s->N;
  a.d = s->d;
  a.bq = s->bq;
  a.nq = ceil_div(s->N, s->bq);
  a.nkv = ceil_div(s->N, s->bkv);
  a.sl2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(s->d)));
  a.sigma = reinterpret_cast<const float*>(ws + L.sigma);
  a.zblk = reinterpret_cast<const float*>(ws + L.zblk);
  a.ztot = reinterpret_cast<const float*>(ws + L.ztot);
  a.phi = phi;
  a.status = reinterpret_cast<int*>(ws + L.status);
  const void* q128 = L.need_hat ? static_cast<const void*>(ws + L.qhat) : q;
  const void* k128 = L.need_hat ? static_cast<const void*>(ws + L.khat) : k;
  a.qsrc = q128;
  if ((e = launch_sparse(a, q128, k128, ws + L.phik, ws + L.v16, ws + L.hs16, ws + L.q8, ws + L.k8, ws + L.v8,
                         st)) != cudaSuccess)
    return cuda_fail(e, "sparse");
  return SLA_OK;
}

}  // namespace

extern "C" {

const char* sla_status_string(sla_status s) {
  switch (s) {
    case SLA_OK: return "SLA_OK";
    case SLA_ERR_INVALID_ARG: return "SLA_ERR_INVALID_ARG";
    case SLA_ERR_UNSUPPORTED: return "SLA_ERR_UNSUPPORTED";
    case SLA_ERR_ALIGNMENT: return "SLA_ERR_ALIGNMENT";
    case SLA_ERR_WORKSPACE: return "SLA_ERR_WORKSPACE";
    case SLA_ERR_CUDA: return "SLA_ERR_CUDA";
    case SLA_ERR_TIMEOUT: return "SLA_ERR_TIMEOUT";
    case SLA_ERR_DEVICE_INDEX: return "SLA_ERR_DEVICE_INDEX";
  }
  return "SLA_ERR_UNKNOWN";
}

const char* sla_last_error_detail(void) { return g_detail; }

int sla_keep_count(double ratio, int n_kv) {
  if (!(ratio > 0.0) || n_kv <= 0) return 0;
  const double k = floor(ratio * n_kv + 0.5);
  if (k < 1.0) return 1;
  if (k > n_kv) return n_kv;
  return static_cast<int>(k);
}

size_t sla_workspace_size(const sla_shape* shape, int mode) {
  if (check_shape(shape) != SLA_OK) return 0;
  const int m = mode & ~SLA_WS_FP8;
  if (m != SLA_MODE_SLA2_TOPK && m != SLA_MODE_SLA_3WAY) return 0;
  return ws_layout(*shape, mode).total;
}

sla_status sla_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || ws_bytes < 256) return arg_fail(SLA_ERR_INVALID_ARG, "ws");
  cudaError_t e = cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SLA_OK : cuda_fail(e, "workspace_init");
}

sla_status sla_route(const sla_shape* shape, const void* q, const void* k, const float* Wq, const float* Wk,
                     int mode, int k_keep, int k_neg, int32_t* kept_idx, int8_t* labels, float* scores_dbg,
                     void* ws, size_t ws_bytes, void* stream) {
  sla_status s = check_shape(shape);
  if (s != SLA_OK) return s;
  const bool kbar_ws = (mode & SLA_ROUTE_KBAR_FROM_WS) != 0;
  mode &= ~SLA_ROUTE_KBAR_FROM_WS;
  if (mode != SLA_MODE_SLA2_TOPK && mode != SLA_MODE_SLA_3WAY) return arg_fail(SLA_ERR_INVALID_ARG, "mode");
  if (kbar_ws && (shape->in_dtype != SLA_BF16 || shape->d != kDPad))
    return arg_fail(SLA_ERR_UNSUPPORTED, "SLA_ROUTE_KBAR_FROM_WS needs bf16 inputs with d = 128");
  if (q == nullptr || k == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "Q or K is null");
  if (!aligned16(q) || !aligned16(k)) return arg_fail(SLA_ERR_ALIGNMENT, "Q, K must be 16-byte aligned");
  if (!aligned16(Wq) || !aligned16(Wk)) return arg_fail(SLA_ERR_ALIGNMENT, "Wq, Wk must be 16-byte aligned");
  const int nkv = ceil_div(shape->N, shape->bkv);
  if (nkv > kMaxNKV) return arg_fail(SLA_ERR_UNSUPPORTED, "router needs n_kv <= 2048");
  if (k_keep < 0 || k_neg < 0 || k_keep + k_neg > nkv) return arg_fail(SLA_ERR_INVALID_ARG, "k_keep/k_neg");
  if (mode == SLA_MODE_SLA2_TOPK && k_neg != 0) return arg_fail(SLA_ERR_INVALID_ARG, "k_neg must be 0 for SLA2");
  if (k_keep > 0 && kept_idx == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "kept_idx is null");
  if ((s = check_ws(shape, SLA_MODE_SLA2_TOPK, ws, ws_bytes)) != SLA_OK) return s;
  const WsLayout L = ws_layout(*shape, SLA_MODE_SLA2_TOPK);
  char* w = static_cast<char*>(ws);
  cudaError_t e = launch_route(*shape, q, k, Wq, Wk, mode, k_keep, k_neg, kept_idx, labels, scores_dbg, L, w,
                               static_cast<cudaStream_t>(stream), 0.0f, nullptr, nullptr,
                               kbar_ws ? reinterpret_cast<const float*>(w + L.kbar) : nullptr);
  return e == cudaSuccess ? SLA_OK : cuda_fail(e, "route");
}

sla_status sla_route_soft(const sla_shape* shape, const void* q, const void* k, const float* Wq, const float* Wk,
                          int k_keep, float tau, float* mask, float* lambda, void* ws, size_t ws_bytes,
                          void* stream) {
  sla_status s = check_shape(shape);
  if (s != SLA_OK) return s;
  if (q == nullptr || k == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "Q or K is null");
  if (mask == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "mask is null");
  if (!(tau > 0.0f) || !(tau < INFINITY)) return arg_fail(SLA_ERR_INVALID_ARG, "tau must be positive and finite");
  if (!aligned16(q) || !aligned16(k)) return arg_fail(SLA_ERR_ALIGNMENT, "Q, K must be 16-byte aligned");
  if (!aligned16(Wq) || !aligned16(Wk)) return arg_fail(SLA_ERR_ALIGNMENT, "Wq, Wk must be 16-byte aligned");
  const int nkv = ceil_div(shape->N, shape->bkv);
  if (nkv > kMaxNKV) return arg_fail(SLA_ERR_UNSUPPORTED, "router needs n_kv <= 2048");
  if (k_keep < 0 || k_keep > nkv) return arg_fail(SLA_ERR_INVALID_ARG, "k_keep");
  if ((s = check_ws(shape, SLA_MODE_SLA2_TOPK, ws, ws_bytes)) != SLA_OK) return s;
  const WsLayout L = ws_layout(*shape, SLA_MODE_SLA2_TOPK);
  cudaError_t e = launch_route(*shape, q, k, Wq, Wk, SLA_MODE_SLA2_TOPK, k_keep, 0, nullptr, nullptr, nullptr, L,
                               static_cast<char*>(ws), static_cast<cudaStream_t>(stream), tau, mask, lambda);
  return e == cudaSuccess ? SLA_OK : cuda_fail(e, "route_soft");
}

sla_status sla_prepare(const sla_shape* shape, const void* k, const void* v, int phi, void* ws, size_t ws_bytes,
                       void* stream) {
  sla_status s = check_shape(shape);
  if (s != SLA_OK) return s;
  if (k == nullptr || v == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "K or V is null");
  if (!aligned16(k) || !aligned16(v)) return arg_fail(SLA_ERR_ALIGNMENT, "K, V must be 16-byte aligned");
  if (phi != SLA_PHI_ELU1 && phi != SLA_PHI_SOFTMAX) return arg_fail(SLA_ERR_INVALID_ARG, "phi");
  if ((s = check_ws(shape, SLA_MODE_SLA2_TOPK, ws, ws_bytes)) != SLA_OK) return s;
  const WsLayout L = ws_layout(*shape, SLA_MODE_SLA2_TOPK);
  cudaError_t e = launch_prepare(*shape, k, v, phi, L, static_cast<char*>(ws), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SLA_OK : cuda_fail(e, "prepare");
}

sla_status sla2_attn_fwd(const sla_shape* shape, const void* q, const void* k, const void* v,
                         const int32_t* kept_idx, int k_keep, const float* alpha, int phi, unsigned flags,
                         void* out, int out_dtype, void* ws, size_t ws_bytes, void* stream) {
  sla_status s = check_shape(shape);
  if (s != SLA_OK) return s;
  if ((s = check_qkv(q, k, v)) != SLA_OK) return s;
  const int nkv = ceil_div(shape->N, shape->bkv);
  if (k_keep < 0 || k_keep > nkv) return arg_fail(SLA_ERR_INVALID_ARG, "k_keep outside [0, n_kv]");
  if (k_keep > 0 && kept_idx == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "kept_idx is null");
  if (alpha == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "alpha is null");
  if (phi != SLA_PHI_ELU1 && phi != SLA_PHI_SOFTMAX) return arg_fail(SLA_ERR_INVALID_ARG, "phi");
  if (flags & ~(SLA_FLAG_PREPARED | SLA_FLAG_FP8 | SLA_FLAG_INT8 | SLA_FLAG_WAIT_TEST))
    return arg_fail(SLA_ERR_INVALID_ARG, "flags");
  if ((flags & SLA_FLAG_FP8) && (flags & SLA_FLAG_INT8))
    return arg_fail(SLA_ERR_INVALID_ARG, "flags: SLA_FLAG_FP8 and SLA_FLAG_INT8 exclude each other");
  if (out == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "out is null");
  if (!aligned16(out)) return arg_fail(SLA_ERR_ALIGNMENT, "out must be 16-byte aligned");
  if (out_dtype != SLA_F32 && out_dtype != SLA_BF16) return arg_fail(SLA_ERR_INVALID_ARG, "out_dtype");
  const int wsmode = SLA_MODE_SLA2_TOPK | ((flags & (SLA_FLAG_FP8 | SLA_FLAG_INT8)) ? SLA_WS_FP8 : 0);
  if ((s = check_ws(shape, wsmode, ws, ws_bytes)) != SLA_OK) return s;
  const WsLayout L = ws_layout(*shape, wsmode);
  SparseArgs a{};
  static const int32_t kNoBlocks = 0;
  a.crit_idx = kept_idx ? kept_idx : &kNoBlocks;  // never read when k_keep == 0
  a.negl_idx = nullptr;
  a.list_stride = k_keep;
  a.crit_max = k_keep;
  a.negl_max = 0;
  a.counts = nullptr;
  a.alpha = alpha;
  a.wproj = nullptr;
  a.out = out;
  a.out_bf16 = out_dtype == SLA_BF16;
  return run_attention(shape, q, k, v, phi, flags, L, static_cast<char*>(ws), static_cast<cudaStream_t>(stream), a);
}

size_t sla2_attn_bwd_workspace_size(const sla_shape* shape) {
  if (shape == nullptr || check_shape(shape) != SLA_OK) return 0;
  return bwd_tc_eligible(*shape) ? bwd_tc_layout(*shape).total : bwd_layout(*shape, false).total;
}

sla_status sla2_attn_bwd(const sla_shape* shape, const void* q, const void* k, const void* v,
                         const int32_t* kept_idx, int k_keep, const float* alpha, int phi, const void* dout,
                         float* dq, float* dk, float* dv, float* dalpha, void* ws, size_t ws_bytes, void* stream) {
  sla_status s = check_shape(shape);
  if (s != SLA_OK) return s;
  if ((s = check_qkv(q, k, v)) != SLA_OK) return s;
  const int nkv = ceil_div(shape->N, shape->bkv);
  if (k_keep < 0 || k_keep > nkv) return arg_fail(SLA_ERR_INVALID_ARG, "k_keep outside [0, n_kv]");
  if (k_keep > 0 && kept_idx == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "kept_idx is null");
  if (alpha == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "alpha is null");
  if (phi != SLA_PHI_ELU1 && phi != SLA_PHI_SOFTMAX) return arg_fail(SLA_ERR_INVALID_ARG, "phi");
  if (dout == nullptr || dq == nullptr || dk == nullptr || dv == nullptr || dalpha == nullptr)
    return arg_fail(SLA_ERR_INVALID_ARG, "dout, dq, dk, dv or dalpha is null");
  if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dalpha))
    return arg_fail(SLA_ERR_ALIGNMENT, "dout, dq, dk, dv, dalpha must be 16-byte aligned");
  if (ws == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "ws is null");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return arg_fail(SLA_ERR_ALIGNMENT, "ws must be 256-byte aligned");
  const bool tc = bwd_tc_eligible(*shape);
  if (ws_bytes < (tc ? bwd_tc_layout(*shape).total : bwd_layout(*shape, false).total))
    return arg_fail(SLA_ERR_WORKSPACE, "ws smaller than sla2_attn_bwd_workspace_size");
  cudaError_t e = tc ? launch_backward_tc(*shape, q, k, v, dout, kept_idx, k_keep, alpha, phi, dq, dk, dv, dalpha,
                                          static_cast<char*>(ws), static_cast<cudaStream_t>(stream))
                     : launch_backward(*shape, q, k, v, dout, kept_idx, k_keep, alpha, phi, dq, dk, dv, dalpha,
                                       static_cast<char*>(ws), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SLA_OK : cuda_fail(e, "backward");
}

size_t sla_attn_bwd_workspace_size(const sla_shape* shape) {
  if (shape == nullptr || check_shape(shape) != SLA_OK) return 0;
  return bwd_layout(*shape, true).total;
}

sla_status sla_attn_bwd(const sla_shape* shape, const void* q, const void* k, const void* v, const int8_t* labels,
                        const void* Wproj, int phi, const void* dout, float* dq, float* dk, float* dv,
                        float* dWproj, void* ws, size_t ws_bytes, void* stream) {
  sla_status s = check_shape(shape);
  if (s != SLA_OK) return s;
  if ((s = check_qkv(q, k, v)) != SLA_OK) return s;
  if (labels == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "labels is null");
  if (Wproj == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "Wproj is null");
  if (phi != SLA_PHI_ELU1 && phi != SLA_PHI_SOFTMAX) return arg_fail(SLA_ERR_INVALID_ARG, "phi");
  if (dout == nullptr || dq == nullptr || dk == nullptr || dv == nullptr || dWproj == nullptr)
    return arg_fail(SLA_ERR_INVALID_ARG, "dout, dq, dk, dv or dWproj is null");
  if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return arg_fail(SLA_ERR_ALIGNMENT, "dout, dq, dk, dv must be 16-byte aligned");
  if (ws == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "ws is null");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return arg_fail(SLA_ERR_ALIGNMENT, "ws must be 256-byte aligned");
  if (ws_bytes < bwd_layout(*shape, true).total)
    return arg_fail(SLA_ERR_WORKSPACE, "ws smaller than sla_attn_bwd_workspace_size");
  cudaError_t e = launch_sla_backward(*shape, q, k, v, dout, labels, Wproj, phi, dq, dk, dv, dWproj,
                                      static_cast<char*>(ws), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SLA_OK : cuda_fail(e, "backward");
}

sla_status sla_attn_fwd(const sla_shape* shape, const void* q, const void* k, const void* v, const int8_t* labels,
                        const void* Wproj, int phi, unsigned flags, void* out, int out_dtype, void* ws,
                        size_t ws_bytes, void* stream) {
  sla_status s = check_shape(shape);
  if (s != SLA_OK) return s;
  if ((s = check_qkv(q, k, v)) != SLA_OK) return s;
  if (labels == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "labels is null");
  if (Wproj == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "Wproj is null");
  if (!aligned16(Wproj)) return arg_fail(SLA_ERR_ALIGNMENT, "Wproj must be 16-byte aligned");
  if (phi != SLA_PHI_ELU1 && phi != SLA_PHI_SOFTMAX) return arg_fail(SLA_ERR_INVALID_ARG, "phi");
  if (flags & ~(SLA_FLAG_PREPARED | SLA_FLAG_FP8 | SLA_FLAG_INT8 | SLA_FLAG_WAIT_TEST))
    return arg_fail(SLA_ERR_INVALID_ARG, "flags");
  if (flags & (SLA_FLAG_FP8 | SLA_FLAG_INT8))
    return arg_fail(SLA_ERR_UNSUPPORTED, "the low-bit sparse branch is built for SLA2 only");
  if (out == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "out is null");
  if (!aligned16(out)) return arg_fail(SLA_ERR_ALIGNMENT, "out must be 16-byte aligned");
  if (out_dtype != SLA_F32 && out_dtype != SLA_BF16) return arg_fail(SLA_ERR_INVALID_ARG, "out_dtype");
  if ((s = check_ws(shape, SLA_MODE_SLA_3WAY, ws, ws_bytes)) != SLA_OK) return s;
  const WsLayout L = ws_layout(*shape, SLA_MODE_SLA_3WAY);
  char* w = static_cast<char*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_labels_to_lists(*shape, labels, L, w, st);
  if (e != cudaSuccess) return cuda_fail(e, "labels");
  const int nkv = ceil_div(shape->N, shape->bkv);
  SparseArgs a{};
  a.crit_idx = reinterpret_cast<const int32_t*>(w + L.lists);
  a.negl_idx = a.crit_idx + nkv;
  a.list_stride = 2LL * nkv;
  a.crit_max = nkv;
  a.negl_max = nkv;
  a.counts = reinterpret_cast<const int32_t*>(w + L.counts);
  a.alpha = nullptr;
  a.wproj = Wproj;
  a.out = out;
  a.out_bf16 = out_dtype == SLA_BF16;
  return run_attention(shape, q, k, v, phi, flags, L, w, st, a);
}

// Device layout of sla2_forward_host: the workspace first (its status word at
// offset 0), then the device copies of the inputs, the kept lists and the output.
struct HostLayout {
  WsLayout ws;
  size_t q = 0, k = 0, v = 0, wq = 0, wk = 0, alpha = 0, kept = 0, out = 0, total = 0;
  size_t in_bytes = 0, out_bytes = 0;
};

static HostLayout host_layout(const sla_shape& s, int k_keep, int out_dtype, unsigned flags) {
  HostLayout H;
  H.ws = ws_layout(s, SLA_MODE_SLA2_TOPK | ((flags & (SLA_FLAG_FP8 | SLA_FLAG_INT8)) ? SLA_WS_FP8 : 0));
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  const size_t nq = static_cast<size_t>(ceil_div(s.N, s.bq));
  const size_t elt = s.in_dtype == SLA_BF16 ? 2 : 4;
  H.in_bytes = BH * s.N * s.d * elt;
  H.out_bytes = BH * s.N * s.d * (out_dtype == SLA_BF16 ? 2 : 4);
  size_t off = H.ws.total;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  H.q = take(H.in_bytes);
  H.k = take(H.in_bytes);
  H.v = take(H.in_bytes);
  H.wq = take(static_cast<size_t>(s.d) * s.d * 4);
  H.wk = take(static_cast<size_t>(s.d) * s.d * 4);
  H.alpha = take(BH * nq * 4);
  H.kept = take(BH * nq * static_cast<size_t>(k_keep > 0 ? k_keep : 0) * 4);
  H.out = take(H.out_bytes);
  H.total = off;
  return H;
}

size_t sla2_forward_host_device_bytes(const sla_shape* shape, int k_keep, int out_dtype, unsigned flags) {
  if (check_shape(shape) != SLA_OK || k_keep < 0 || k_keep > ceil_div(shape->N, shape->bkv)) return 0;
  if (out_dtype != SLA_F32 && out_dtype != SLA_BF16) return 0;
  return host_layout(*shape, k_keep, out_dtype, flags).total;
}

sla_status sla2_forward_host(const sla_shape* shape, const void* q, const void* k, const void* v, const float* Wq,
                             const float* Wk, const float* alpha, int k_keep, int phi, unsigned flags, void* out,
                             int out_dtype, int32_t* kept_out, void* dev, size_t dev_bytes, void* stream) {
  sla_status s = check_shape(shape);
  if (s != SLA_OK) return s;
  if (q == nullptr || k == nullptr || v == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "Q, K or V is null");
  if (alpha == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "alpha is null");
  if (out == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "out is null");
  if (out_dtype != SLA_F32 && out_dtype != SLA_BF16) return arg_fail(SLA_ERR_INVALID_ARG, "out_dtype");
  if (phi != SLA_PHI_ELU1 && phi != SLA_PHI_SOFTMAX) return arg_fail(SLA_ERR_INVALID_ARG, "phi");
  if (flags & ~(SLA_FLAG_FP8 | SLA_FLAG_INT8))
    return arg_fail(SLA_ERR_INVALID_ARG, "flags (only SLA_FLAG_FP8 or SLA_FLAG_INT8 is accepted)");
  const int nkv = ceil_div(shape->N, shape->bkv);
  if (nkv > kMaxNKV) return arg_fail(SLA_ERR_UNSUPPORTED, "router needs n_kv <= 2048");
  if (k_keep < 0 || k_keep > nkv) return arg_fail(SLA_ERR_INVALID_ARG, "k_keep outside [0, n_kv]");
  if (dev == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "dev is null");
  if ((reinterpret_cast<uintptr_t>(dev) & 255u) != 0) return arg_fail(SLA_ERR_ALIGNMENT, "dev must be 256-byte aligned");
  const HostLayout H = host_layout(*shape, k_keep, out_dtype, flags);
  if (dev_bytes < H.total) return arg_fail(SLA_ERR_WORKSPACE, "dev smaller than sla2_forward_host_device_bytes");
  char* d = static_cast<char*>(dev);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t nq = static_cast<size_t>(ceil_div(shape->N, shape->bq));
  const size_t BH = static_cast<size_t>(shape->B) * shape->H;
  const size_t wbytes = static_cast<size_t>(shape->d) * shape->d * 4;
  // one plain asynchronous copy per buffer (pinned host memory lets them overlap the host)
  struct { void* dst; const void* src; size_t n; } in[] = {
      {d + H.q, q, H.in_bytes}, {d + H.k, k, H.in_bytes}, {d + H.v, v, H.in_bytes},
      {d + H.wq, Wq, Wq ? wbytes : 0}, {d + H.wk, Wk, Wk ? wbytes : 0}, {d + H.alpha, alpha, BH * nq * 4}};
  for (const auto& c : in) {
    if (c.n == 0) continue;
    cudaError_t e = cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
  }
  const float* wq_d = Wq ? reinterpret_cast<const float*>(d + H.wq) : nullptr;
  const float* wk_d = Wk ? reinterpret_cast<const float*>(d + H.wk) : nullptr;
  int32_t* kept_d = reinterpret_cast<int32_t*>(d + H.kept);
  // bf16, d = 128: the prepass writes the key-block means and the router reuses them
  const bool kbar_first = shape->in_dtype == SLA_BF16 && shape->d == kDPad;
  const size_t wsb = H.ws.total;
  if (kbar_first && (s = sla_prepare(shape, d + H.k, d + H.v, phi, d, wsb, stream)) != SLA_OK) return s;
  if ((s = sla_route(shape, d + H.q, d + H.k, wq_d, wk_d, SLA_MODE_SLA2_TOPK | (kbar_first ? SLA_ROUTE_KBAR_FROM_WS : 0),
                     k_keep, 0, kept_d, nullptr, nullptr, d, wsb, stream)) != SLA_OK)
    return s;
  if (!kbar_first && (s = sla_prepare(shape, d + H.k, d + H.v, phi, d, wsb, stream)) != SLA_OK) return s;
  if ((s = sla2_attn_fwd(shape, d + H.q, d + H.k, d + H.v, kept_d, k_keep, reinterpret_cast<const float*>(d + H.alpha),
                         phi, SLA_FLAG_PREPARED | (flags & (SLA_FLAG_FP8 | SLA_FLAG_INT8)), d + H.out, out_dtype, d,
                         wsb, stream)) !=
      SLA_OK)
    return s;
  cudaError_t e = cudaMemcpyAsync(out, d + H.out, H.out_bytes, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
  if (kept_out != nullptr && k_keep > 0) {
    e = cudaMemcpyAsync(kept_out, kept_d, BH * nq * k_keep * 4, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
  }
  return SLA_OK;
}

sla_status sla_read_device_status(void* ws, void* stream) {
  if (ws == nullptr) return arg_fail(SLA_ERR_INVALID_ARG, "ws is null");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "synchronize");
  int code = 0;
  e = cudaMemcpy(&code, ws, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  e = cudaMemset(ws, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  return static_cast<sla_status>(code);
}

}  // extern "C"
