// route_noalloc.cu -- the router for callers that cannot hand the library a
// device workspace.
//
// Some callers cannot allocate device memory at the point where they route:
// code running inside another framework's memory manager that forbids
// allocations outside its own pools, or a host thread that must not call
// cudaMalloc because of the implicit synchronisation and capture restrictions
// that come with it.  sla_route_noalloc serves them: it runs the same three
// router kernels as sla_route, but their scratch (pooled and projected block
// means) lives in a fixed array compiled into the library, so the call
// allocates nothing.
//
// The array is file-scope device memory of a fixed size: every GPU that loads
// libsla holds it until the process exits.  Its device address is looked up
// once per device, on that device's first call (with the device current).
// All calls share the one array, so calls that overlap on the GPU (different
// streams, or several host threads) race on it.  The router kernels write
// every scratch element before reading it, so nothing needs clearing between
// calls.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "sla_internal.h"
#include "sla_kernels.h"

namespace sla {

// 16 MiB: projected block means of Q and K, B*H*(n_q + n_kv)*d floats plus
// alignment (the 1.3B-shape workload needs 4.7 MB).
constexpr size_t kNoAllocScratchBytes = 16u << 20;

static __device__ __align__(256) char g_route_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
char* g_scratch[kMaxDevices] = {};

// Device address of g_route_scratch on the current device (set-up on first use).
cudaError_t scratch_on_current_device(char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    g_scratch[dev] = static_cast<char*>(p);
  }
  *out = g_scratch[dev];
  return cudaSuccess;
}

// Router scratch laid out from offset 0 with the workspace's 256-byte rounding.
WsLayout route_scratch_layout(const sla_shape& s, size_t* bytes) {
  WsLayout L;
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  const size_t nq = static_cast<size_t>(ceil_div(s.N, s.bq)), nkv = static_cast<size_t>(ceil_div(s.N, s.bkv));
  size_t off = 0;
  L.qt = off;
  off = align256(off + BH * nq * s.d * 4);
  L.kt = off;
  off = align256(off + BH * static_cast<size_t>(kt_stride(static_cast<int>(nkv))) * s.d * 4);
  *bytes = off;
  return L;
}

}  // namespace

}  // namespace sla

using namespace sla;

extern "C" sla_status sla_route_noalloc(const sla_shape* shape, const void* q, const void* k, const float* Wq,
                                        const float* Wk, int mode, int k_keep, int k_neg, int32_t* kept_idx,
                                        int8_t* labels, float* scores_dbg, void* stream) {
  // Same argument rules as sla_route; everything is checked before any launch.
  if (shape == nullptr) return SLA_ERR_INVALID_ARG;
  const sla_shape& s = *shape;
  if (s.B < 1 || s.H < 1 || s.N < 1 || s.d < 1 || s.bq < 1 || s.bkv < 1) return SLA_ERR_INVALID_ARG;
  if (s.in_dtype != SLA_F32 && s.in_dtype != SLA_BF16) return SLA_ERR_INVALID_ARG;
  if (s.d % 8 != 0 || s.d > kDPad || (s.bq != 64 && s.bq != 128) || s.bkv != kBlockKV || s.N > kMaxN ||
      static_cast<long long>(s.B) * s.H > 65535)
    return SLA_ERR_UNSUPPORTED;
  if (mode != SLA_MODE_SLA2_TOPK && mode != SLA_MODE_SLA_3WAY) return SLA_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr) return SLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(k) & 15u) ||
      (reinterpret_cast<uintptr_t>(Wq) & 15u) || (reinterpret_cast<uintptr_t>(Wk) & 15u))
    return SLA_ERR_ALIGNMENT;
  const int nkv = ceil_div(s.N, s.bkv);
  if (nkv > kMaxNKV) return SLA_ERR_UNSUPPORTED;
  if (k_keep < 0 || k_neg < 0 || k_keep + k_neg > nkv) return SLA_ERR_INVALID_ARG;
  if (mode == SLA_MODE_SLA2_TOPK && k_neg != 0) return SLA_ERR_INVALID_ARG;
  if (k_keep > 0 && kept_idx == nullptr) return SLA_ERR_INVALID_ARG;
  size_t need = 0;
  const WsLayout L = route_scratch_layout(s, &need);
  if (need > kNoAllocScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "sla_route_noalloc: this shape needs %zu bytes of router scratch, more than the built-in %zu",
             need, kNoAllocScratchBytes);
    set_error_detail(msg);
    return SLA_ERR_WORKSPACE;
  }
  char* scratch = nullptr;
  cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) {
    set_error_detail(cudaGetErrorString(e));
    return SLA_ERR_CUDA;
  }
  e = launch_route(s, q, k, Wq, Wk, mode, k_keep, k_neg, kept_idx, labels, scores_dbg, L, scratch,
                   static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    set_error_detail(cudaGetErrorString(e));
    return SLA_ERR_CUDA;
  }
  return SLA_OK;
}
