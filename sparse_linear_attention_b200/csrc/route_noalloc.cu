// route_noalloc.cu -- the router for callers that cannot hand the library a
// device workspace.
//
// Some callers cannot allocate device memory at the point where they route:
// code running inside another framework's memory manager that forbids
// allocations outside its own pools, or a host thread that must not call
// cudaMalloc because of the implicit synchronisation and capture restrictions
// that come with it.  sla_route_noalloc serves them: it runs the same two
// router kernels as sla_route, but their scratch (the projected block means
// of Q and K) lives in a fixed array compiled into the library, so the call
// allocates nothing.
//
// The array is file-scope device memory of a fixed size: every GPU that loads
// libsla holds it until the process exits.  Its device address is looked up
// with cudaGetSymbolAddress on the first call in each CUDA context (with the
// device current) and cached together with that context's unique id; a call
// that finds a different context current (after cudaDeviceReset, or once the
// primary context was destroyed and made again, which reloads the module and
// may move the array) looks the address up again instead of using a stale one.
// All calls share the one array, so calls that overlap on the GPU (different
// streams, or several host threads) race on it.  Nothing in it needs clearing
// between calls: the router kernels write every scratch element whose value
// reaches a result before reading it.  The only elements read without being
// written are the up to three padding columns of the key means (their rows
// are padded to a multiple of four keys); they hold what an earlier call left
// there, and the scores computed from them are dropped.
#include <cudaTypedefs.h>
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
struct Cached {
  char* ptr = nullptr;
  unsigned long long ctx_id = 0;  // the context the address belongs to
};
Cached g_scratch[kMaxDevices];

// Unique id of the CUDA context current on this thread (driver API, looked up
// through the runtime so that libsla links only cudart).  Returns false when
// no valid context is current.
bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f1, 4000, cudaEnableDefault, &q1) == cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f1);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f2, 12000, cudaEnableDefault, &q2) == cudaSuccess &&
        q2 == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f2);
    looked_up = true;
  }
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_route_scratch in the current device's context.  Set-up:
// cudaGetSymbolAddress, with the device current, the first time a context is
// seen (it also creates the primary context if none is current yet).
cudaError_t scratch_on_current_device(char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  Cached& c = g_scratch[dev];
  unsigned long long id = 0;
  if (c.ptr != nullptr && current_context_id(&id) && id == c.ctx_id) {
    *out = c.ptr;
    return cudaSuccess;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_route_scratch);
  if (e != cudaSuccess) return e;
  if (!current_context_id(&id)) id = 0;  // unknown context: looked up again on the next call
  c.ptr = static_cast<char*>(p);
  c.ctx_id = id;
  *out = c.ptr;
  return cudaSuccess;
}

sla_status reject(sla_status s, const char* what) {
  char msg[200];
  snprintf(msg, sizeof(msg), "sla_route_noalloc: %s", what);
  set_error_detail(msg);
  return s;
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
  if (shape == nullptr) return reject(SLA_ERR_INVALID_ARG, "shape is null");
  const sla_shape& s = *shape;
  if (s.B < 1 || s.H < 1 || s.N < 1 || s.d < 1 || s.bq < 1 || s.bkv < 1)
    return reject(SLA_ERR_INVALID_ARG, "shape sizes must be positive");
  if (s.in_dtype != SLA_F32 && s.in_dtype != SLA_BF16) return reject(SLA_ERR_INVALID_ARG, "in_dtype");
  if (s.d % 8 != 0 || s.d > kDPad) return reject(SLA_ERR_UNSUPPORTED, "d must be a multiple of 8, <= 128");
  if (s.bq != 64 && s.bq != 128) return reject(SLA_ERR_UNSUPPORTED, "bq must be 64 or 128");
  if (s.bkv != kBlockKV) return reject(SLA_ERR_UNSUPPORTED, "bkv must be 64");
  if (s.N > kMaxN) return reject(SLA_ERR_UNSUPPORTED, "N > 131072");
  if (static_cast<long long>(s.B) * s.H > 65535) return reject(SLA_ERR_UNSUPPORTED, "B*H > 65535");
  if (mode & SLA_ROUTE_KBAR_FROM_WS)
    return reject(SLA_ERR_INVALID_ARG,
                  "SLA_ROUTE_KBAR_FROM_WS is not supported: there is no workspace holding key-block means");
  if (mode != SLA_MODE_SLA2_TOPK && mode != SLA_MODE_SLA_3WAY) return reject(SLA_ERR_INVALID_ARG, "mode");
  if (q == nullptr || k == nullptr) return reject(SLA_ERR_INVALID_ARG, "Q or K is null");
  if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(k) & 15u))
    return reject(SLA_ERR_ALIGNMENT, "Q, K must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(Wq) & 15u) || (reinterpret_cast<uintptr_t>(Wk) & 15u))
    return reject(SLA_ERR_ALIGNMENT, "Wq, Wk must be 16-byte aligned");
  const int nkv = ceil_div(s.N, s.bkv);
  if (nkv > kMaxNKV) return reject(SLA_ERR_UNSUPPORTED, "router needs n_kv <= 2048");
  if (k_keep < 0 || k_neg < 0 || k_keep + k_neg > nkv) return reject(SLA_ERR_INVALID_ARG, "k_keep/k_neg");
  if (mode == SLA_MODE_SLA2_TOPK && k_neg != 0) return reject(SLA_ERR_INVALID_ARG, "k_neg must be 0 for SLA2");
  if (k_keep > 0 && kept_idx == nullptr) return reject(SLA_ERR_INVALID_ARG, "kept_idx is null");
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
  if (e != cudaSuccess) return reject(SLA_ERR_CUDA, cudaGetErrorString(e));
  e = launch_route(s, q, k, Wq, Wk, mode, k_keep, k_neg, kept_idx, labels, scores_dbg, L, scratch,
                   static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return reject(SLA_ERR_CUDA, cudaGetErrorString(e));
  return SLA_OK;
}
