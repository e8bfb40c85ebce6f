// labels.cu -- SLA labels (+1 critical, 0 marginal, -1 negligible) to
// per-row block lists for the attention kernel ("SLA: Beyond Sparsity in
// Diffusion Transformers …" (papernotes.org) 关键设计 2).
//
// One warp per (b,h, query block) row: critical and negligible block indices
// in ascending order, and their counts.  A label outside {-1, 0, 1} sets
// SLA_ERR_DEVICE_INDEX in the status word (the block is then treated as
// marginal).
#include <stdint.h>

#include "sla_device.cuh"
#include "sla_internal.h"
#include "sla_kernels.h"

namespace sla {

namespace {

__global__ void __launch_bounds__(256) labels_to_lists_kernel(const int8_t* __restrict__ labels,
                                                              int32_t* __restrict__ lists,
                                                              int32_t* __restrict__ counts, long long rows,
                                                              int nkv, int* status) {
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int8_t* lab = labels + row * nkv;
  int32_t* crit = lists + row * 2 * nkv;
  int32_t* negl = crit + nkv;
  int nc = 0, nn = 0;
  for (int j0 = 0; j0 < nkv; j0 += 32) {
    const int j = j0 + lane;
    const int l = j < nkv ? lab[j] : 0;
    if (l < -1 || l > 1) report_error(status, SLA_ERR_DEVICE_INDEX);
    const uint32_t mc = __ballot_sync(0xffffffffu, l == 1);
    const uint32_t mn = __ballot_sync(0xffffffffu, l == -1);
    const uint32_t below = (1u << lane) - 1u;
    if (l == 1) crit[nc + __popc(mc & below)] = j;
    if (l == -1) negl[nn + __popc(mn & below)] = j;
    nc += __popc(mc);
    nn += __popc(mn);
  }
  if (lane == 0) {
    counts[2 * row] = nc;
    counts[2 * row + 1] = nn;
  }
}

}  // namespace

cudaError_t launch_labels_to_lists(const sla_shape& s, const int8_t* labels, int32_t* lists, int32_t* counts,
                                   int* status, cudaStream_t st) {
  const long long rows = static_cast<long long>(s.B) * s.H * ceil_div(s.N, s.bq);
  const int nkv = ceil_div(s.N, s.bkv);
  labels_to_lists_kernel<<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, st>>>(labels, lists, counts, rows,
                                                                                        nkv, status);
  return cudaGetLastError();
}

cudaError_t launch_labels_to_lists(const sla_shape& s, const int8_t* labels, const WsLayout& L, char* ws,
                                   cudaStream_t st) {
  return launch_labels_to_lists(s, labels, reinterpret_cast<int32_t*>(ws + L.lists),
                                reinterpret_cast<int32_t*>(ws + L.counts), reinterpret_cast<int*>(ws + L.status), st);
}

}  // namespace sla
