// route.cu -- the router: block mean-pooling, learnable projections, block
// scores and hard selection.
//
// Follows "SLA2 深度解读 …" (jefxiong.cn) §05 (pool(Q), pool(K), proj_q, proj_k,
// P_c = proj_q(Qbar) proj_k(Kbar)^T, M_c = Top-k(k%, P_c)) and "SLA: Beyond
// Sparsity in Diffusion Transformers …" (papernotes.org) 关键设计 2 (three
// labels: top k_h critical, bottom k_l negligible, rest marginal).
//
// Every floating-point step is a single IEEE round-to-nearest operation in a
// fixed order (__fadd_rn / __fmul_rn / __fdiv_rn never contract into FMA), so
// the selected blocks are reproducible bit for bit on any implementation that
// follows the same order:
//   pooled mean : tokens ascending from +0.0, then divide by the count
//   projection  : y[c] = sum_e fl(x[e] * W[e][c]), e ascending, from +0.0
//   score       : s[i][j] = sum_c fl(qt[i][c] * kt[j][c]), c ascending, from +0.0
// The ranking is (score descending, block index ascending).
#include <cuda_bf16.h>
#include <math_constants.h>
#include <stdint.h>

#include "sla_device.cuh"
#include "sla_internal.h"
#include "sla_kernels.h"

namespace sla {

// ---------------------------------------------------------------- pooling
// One thread per (head, block, 16-byte channel unit); tokens summed in
// ascending order.  The grid's y index selects Q (0) or K (1).
template <typename T>
__global__ void __launch_bounds__(256) pool_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                   float* __restrict__ qbar, float* __restrict__ kbar,
                                                   int BH, int N, int d, int bq, int bkv) {
  constexpr int VPU = 16 / sizeof(T);  // channels per 16-byte unit
  const bool isK = blockIdx.y == 1;
  const T* x = isK ? k : q;
  float* xbar = isK ? kbar : qbar;
  const int b = isK ? bkv : bq;
  const int nb = (N + b - 1) / b;
  const int upr = d / VPU;
  const long long total = static_cast<long long>(BH) * nb * upr;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int u = static_cast<int>(idx % upr);
  const int blk = static_cast<int>((idx / upr) % nb);
  const long long bh = idx / (static_cast<long long>(upr) * nb);
  const int start = blk * b;
  const int cnt = min(b, N - start);
  const uint4* src = reinterpret_cast<const uint4*>(x + (bh * N + start) * d) + u;
  const int stride = d / VPU;  // uint4 per token row
  float acc[VPU];
#pragma unroll
  for (int c = 0; c < VPU; ++c) acc[c] = 0.0f;
  for (int t0 = 0; t0 < cnt; t0 += 8) {
    uint4 buf[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (t0 + i < cnt) buf[i] = __ldg(src + static_cast<long long>(t0 + i) * stride);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (t0 + i < cnt) {
        const T* e = reinterpret_cast<const T*>(&buf[i]);
#pragma unroll
        for (int c = 0; c < VPU; ++c) acc[c] = __fadd_rn(acc[c], static_cast<float>(e[c]));
      }
    }
  }
  const float fc = static_cast<float>(cnt);
  float* dst = xbar + (bh * nb + blk) * d + u * VPU;
#pragma unroll
  for (int c = 0; c < VPU; ++c) dst[c] = __fdiv_rn(acc[c], fc);
}

// ---------------------------------------------------------------- projection
// xt^T[bh][c][r] = sum_e fl(xbar[bh][r][e] * W[e][c]) (or xbar itself when W is
// null), written channel-major so the score kernel reads it coalesced.
// Block: 256 threads, 64 rows of one head x all d output channels; thread
// (ty, tx) owns rows 4ty..4ty+3 and channels 8tx..8tx+7.  The sum over e runs
// in ascending order for every output, as specified.
constexpr int kProjRows = 64;

__global__ void __launch_bounds__(256) project_kernel(const float* __restrict__ qbar,
                                                      const float* __restrict__ kbar,
                                                      const float* __restrict__ Wq,
                                                      const float* __restrict__ Wk, float* __restrict__ qtT,
                                                      float* __restrict__ ktT, int nq, int nkv, int d) {
  const bool isK = blockIdx.z == 1;
  const float* xbar = isK ? kbar : qbar;
  const float* W = isK ? Wk : Wq;
  float* xtT = isK ? ktT : qtT;
  const int nrows = isK ? nkv : nq;
  const int r0 = blockIdx.x * kProjRows;
  if (r0 >= nrows) return;
  const long long bh = blockIdx.y;
  extern __shared__ __align__(16) float psm[];
  float* xs = psm;                     // [d][64]: xs[e][r] = xbar[r0 + r][e]
  float* ws = psm + kDPad * kProjRows; // [d][128]: W[e][c]
  const int tid = threadIdx.x;
  // rows: float4 along e, one row per thread in a group of 64 -> transposed store
  for (int i = tid; i < kProjRows * (d / 4); i += 256) {
    const int r = i % kProjRows, e4 = i / kProjRows;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < nrows) v = *reinterpret_cast<const float4*>(xbar + (bh * nrows + r0 + r) * d + 4 * e4);
    xs[(4 * e4 + 0) * kProjRows + r] = v.x;
    xs[(4 * e4 + 1) * kProjRows + r] = v.y;
    xs[(4 * e4 + 2) * kProjRows + r] = v.z;
    xs[(4 * e4 + 3) * kProjRows + r] = v.w;
  }
  if (W != nullptr)
    for (int i = tid; i < d * (d / 4); i += 256) cp_async16(ws + (i / (d / 4)) * kDPad + 4 * (i % (d / 4)), W + 4 * i);
  cp_async_wait_all();
  __syncthreads();
  const int ty = tid / 16, tx = tid % 16;
  if (8 * tx >= d) return;
  float acc[4][8];
  if (W == nullptr) {
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) acc[a][b] = xs[(8 * tx + b) * kProjRows + 4 * ty + a];
  } else {
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) acc[a][b] = 0.0f;
    for (int e = 0; e < d; ++e) {
      const float4 xv = *reinterpret_cast<const float4*>(xs + e * kProjRows + 4 * ty);
      const float4 w0 = *reinterpret_cast<const float4*>(ws + e * kDPad + 8 * tx);
      const float4 w1 = *reinterpret_cast<const float4*>(ws + e * kDPad + 8 * tx + 4);
      const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
      const float wb[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = __fadd_rn(acc[a][b], __fmul_rn(xa[a], wb[b]));
    }
  }
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    float* dst = xtT + (bh * d + 8 * tx + b) * nrows + r0 + 4 * ty;
#pragma unroll
    for (int a = 0; a < 4; ++a)
      if (r0 + 4 * ty + a < nrows) dst[a] = acc[a][b];
  }
}

// ---------------------------------------------------------------- scores + selection
// Block: 256 threads, 16 query blocks of one head.  Scores for the 16 rows
// are built in shared memory chunk by chunk (128 key blocks per chunk, each
// thread 2 rows x 4 key blocks), then each warp selects for 2 rows.
constexpr int kScoreRows = 16;
constexpr int kScoreKeys = 128;

struct Cand {
  float s;
  int j;
};

// a ranks before b in (score desc, index asc)
__device__ __forceinline__ bool ranks_before(float sa, int ja, float sb, int jb) {
  return sa > sb || (sa == sb && ja < jb);
}

__device__ __forceinline__ Cand warp_best(Cand c, bool top) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float s2 = __shfl_xor_sync(0xffffffffu, c.s, o);
    const int j2 = __shfl_xor_sync(0xffffffffu, c.j, o);
    const bool take = top ? ranks_before(s2, j2, c.s, c.j) : ranks_before(c.s, c.j, s2, j2);
    if (take) {
      c.s = s2;
      c.j = j2;
    }
  }
  return c;
}

// Best unmarked element of this lane (j = lane + 32 t); `top` picks the
// first in rank order, otherwise the last.
__device__ __forceinline__ Cand lane_best(const float* row, int nkv, int lane, uint64_t excl, bool top) {
  Cand c;
  c.s = top ? -CUDART_INF_F : CUDART_INF_F;
  c.j = top ? INT32_MAX : -1;
  for (int t = 0; lane + 32 * t < nkv; ++t) {
    if ((excl >> t) & 1ull) continue;
    const int j = lane + 32 * t;
    const float s = row[j];
    const bool take = top ? ranks_before(s, j, c.s, c.j) : ranks_before(c.s, c.j, s, j);
    if (take) {
      c.s = s;
      c.j = j;
    }
  }
  return c;
}

__global__ void __launch_bounds__(256) score_select_kernel(const float* __restrict__ qtT,
                                                           const float* __restrict__ ktT, int nq, int nkv,
                                                           int d, int mode, int k_keep, int k_neg,
                                                           int32_t* __restrict__ kept_idx,
                                                           int8_t* __restrict__ labels,
                                                           float* __restrict__ scores_dbg) {
  extern __shared__ __align__(16) float sm[];
  float* qs = sm;                            // [d][16]
  float* ks = qs + kDPad * kScoreRows;       // [d][128]
  float* sc = ks + kDPad * kScoreKeys;       // [16][nkv]
  const long long bh = blockIdx.y;
  const int r0 = blockIdx.x * kScoreRows;
  const int tid = threadIdx.x;
  for (int i = tid; i < d * kScoreRows; i += 256) {
    const int c = i / kScoreRows, r = i % kScoreRows;
    qs[i] = (r0 + r < nq) ? qtT[(bh * d + c) * nq + r0 + r] : 0.0f;
  }
  const bool vec_ok = (nkv % 4) == 0;  // rows of ktT 16-byte aligned
  const int ty = tid / 32;  // rows 2*ty, 2*ty+1
  const int tx = tid % 32;  // key blocks 4*tx .. 4*tx+3 of the chunk
  for (int j0 = 0; j0 < nkv; j0 += kScoreKeys) {
    __syncthreads();  // previous chunk's ks reads done (and qs ready on the first pass)
    if (vec_ok && j0 + kScoreKeys <= nkv) {
      for (int i = tid; i < d * (kScoreKeys / 4); i += 256) {
        const int c = i / (kScoreKeys / 4), j4 = i % (kScoreKeys / 4);
        cp_async16(ks + c * kScoreKeys + 4 * j4, ktT + (bh * d + c) * nkv + j0 + 4 * j4);
      }
      cp_async_wait_all();
    } else {
#pragma unroll 8
      for (int i = tid; i < d * kScoreKeys; i += 256) {
        const int c = i / kScoreKeys, j = i % kScoreKeys;
        ks[i] = (j0 + j < nkv) ? ktT[(bh * d + c) * nkv + j0 + j] : 0.0f;
      }
    }
    __syncthreads();
    float acc[2][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
    for (int c = 0; c < d; ++c) {
      const float2 qv = *reinterpret_cast<const float2*>(qs + c * kScoreRows + 2 * ty);
      const float4 kv = *reinterpret_cast<const float4*>(ks + c * kScoreKeys + 4 * tx);
      const float qa[2] = {qv.x, qv.y};
      const float kb[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = __fadd_rn(acc[a][b], __fmul_rn(qa[a], kb[b]));
    }
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int j = j0 + 4 * tx + b;
        if (j < nkv) sc[(2 * ty + a) * nkv + j] = acc[a][b];
      }
  }
  __syncthreads();

  const int lane = tid % 32, warp = tid / 32;
  for (int rr = 0; rr < 2; ++rr) {
    const int r = warp * 2 + rr;
    const int row = r0 + r;
    if (row >= nq) break;
    const float* srow = sc + r * nkv;
    const long long grow = bh * nq + row;
    uint64_t top = 0, bot = 0;
    Cand mine = lane_best(srow, nkv, lane, top, true);
    for (int it = 0; it < k_keep; ++it) {
      const Cand w = warp_best(mine, true);
      if ((w.j & 31) == lane) {
        top |= 1ull << (w.j >> 5);
        mine = lane_best(srow, nkv, lane, top, true);
      }
    }
    if (mode == SLA_MODE_SLA_3WAY && k_neg > 0) {
      mine = lane_best(srow, nkv, lane, top, false);
      for (int it = 0; it < k_neg; ++it) {
        const Cand w = warp_best(mine, false);
        if ((w.j & 31) == lane) {
          bot |= 1ull << (w.j >> 5);
          mine = lane_best(srow, nkv, lane, top | bot, false);
        }
      }
    }
    // kept indices in ascending order
    int base = 0;
    for (int t = 0; 32 * t < nkv; ++t) {
      const int j = lane + 32 * t;
      const bool s = (j < nkv) && ((top >> t) & 1ull);
      const uint32_t m = __ballot_sync(0xffffffffu, s);
      if (s) kept_idx[grow * k_keep + base + __popc(m & ((1u << lane) - 1u))] = j;
      base += __popc(m);
      if (j < nkv) {
        if (labels) labels[grow * nkv + j] = s ? 1 : (((bot >> t) & 1ull) ? -1 : 0);
        if (scores_dbg) scores_dbg[grow * nkv + j] = srow[j];
      }
    }
  }
}

// ---------------------------------------------------------------- launchers

cudaError_t launch_route(const sla_shape& s, const void* q, const void* k, const float* Wq, const float* Wk,
                         int mode, int k_keep, int k_neg, int32_t* kept_idx, int8_t* labels,
                         float* scores_dbg, const WsLayout& L, char* ws, cudaStream_t st) {
  const int BH = s.B * s.H;
  const int nq = ceil_div(s.N, s.bq), nkv = ceil_div(s.N, s.bkv);
  float* qbar = reinterpret_cast<float*>(ws + L.qbar);
  float* kbar = reinterpret_cast<float*>(ws + L.kbar);
  float* qtT = reinterpret_cast<float*>(ws + L.qt);
  float* ktT = reinterpret_cast<float*>(ws + L.kt);
  {
    const int vpu = s.in_dtype == SLA_BF16 ? 8 : 4;
    const long long nthr = static_cast<long long>(BH) * nq * (s.d / vpu);
    const long long nthr_k = static_cast<long long>(BH) * nkv * (s.d / vpu);
    const long long mx = nthr > nthr_k ? nthr : nthr_k;
    dim3 grid(static_cast<unsigned>((mx + 255) / 256), 2);
    if (s.in_dtype == SLA_BF16)
      pool_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                                        static_cast<const __nv_bfloat16*>(k), qbar, kbar, BH,
                                                        s.N, s.d, s.bq, s.bkv);
    else
      pool_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                                qbar, kbar, BH, s.N, s.d, s.bq, s.bkv);
  }
  {
    const size_t psmem = static_cast<size_t>(kDPad) * (kProjRows + kDPad) * 4;
    cudaError_t e = cudaFuncSetAttribute(project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(psmem));
    if (e != cudaSuccess) return e;
    dim3 grid(ceil_div(nkv > nq ? nkv : nq, kProjRows), BH, 2);
    project_kernel<<<grid, 256, psmem, st>>>(qbar, kbar, Wq, Wk, qtT, ktT, nq, nkv, s.d);
  }
  {
    const size_t smem = (kDPad * kScoreRows + kDPad * kScoreKeys + static_cast<size_t>(kScoreRows) * nkv) * 4;
    cudaError_t e = cudaFuncSetAttribute(score_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(ceil_div(nq, kScoreRows), BH);
    score_select_kernel<<<grid, 256, smem, st>>>(qtT, ktT, nq, nkv, s.d, mode, k_keep, k_neg, kept_idx, labels,
                                                 scores_dbg);
  }
  return cudaGetLastError();
}

}  // namespace sla
