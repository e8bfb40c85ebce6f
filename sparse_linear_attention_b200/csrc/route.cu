// route.cu -- the router: block mean-pooling, learnable projections, block
// scores and hard selection.
//
// Follows "SLA2 深度解读 …" (jefxiong.cn) §05 (pool(Q), pool(K), proj_q, proj_k,
// P_c = proj_q(Qbar) proj_k(Kbar)^T, M_c = Top-k(k%, P_c)) and "SLA: Beyond
// Sparsity in Diffusion Transformers …" (papernotes.org) 关键设计 2 (three
// labels: top k_h critical, bottom k_l negligible, rest marginal).
//
// Every floating-point step is a single IEEE round-to-nearest operation in a
// fixed order (__fadd_rn / __fdiv_rn / __fmaf_rn), so the selected blocks are
// reproducible bit for bit on any implementation that follows the same order
// (pooling and projection run in one kernel, the means staying in shared
// memory):
//   pooled mean : tokens ascending from +0.0, then divide by the count
//   projection  : y[c] = fma(x[e], W[e][c], y[c]), e ascending, from +0.0
//   score       : s[i][j] = fma(qt[i][c], kt[j][c], s[i][j]), c ascending, from +0.0
// The ranking is (score descending, block index ascending).
#include <cuda_bf16.h>
#include <math_constants.h>
#include <stdint.h>

#include "sla_device.cuh"
#include "sla_internal.h"
#include "sla_kernels.h"

namespace sla {

// ---------------------------------------------------------------- pooling + projection
// One block per kPPRows blocks (rows) of one head and one of Q (grid z = 0) or
// K (z = 1): the block means go to shared memory (tokens ascending from +0.0,
// then one division) and are projected at once (e ascending, one rounding
// per multiply-add), so the projection's arithmetic
// runs under the pooling's HBM traffic and the means never leave the chip.
constexpr int kPPRows = 16;

template <typename T>
__global__ void __launch_bounds__(256) pool_project_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                           const float* __restrict__ Wq,
                                                           const float* __restrict__ Wk,
                                                           float* __restrict__ qtT, float* __restrict__ ktT,
                                                           int N, int d, int bq, int bkv, int kstride) {
  constexpr int VPU = 16 / sizeof(T);  // channels per 16-byte unit
  const bool isK = blockIdx.z == 1;
  const T* x = isK ? k : q;
  const float* W = isK ? Wk : Wq;
  float* xtT = isK ? ktT : qtT;
  const int b = isK ? bkv : bq;
  const int nrows = (N + b - 1) / b;
  const int r0 = blockIdx.x * kPPRows;
  if (r0 >= nrows) return;
  const long long bh = blockIdx.y;
  __shared__ __align__(16) float xs[kPPRows][kDPad];
  const int tid = threadIdx.x;
  const int upr = d / VPU;
  for (int i = tid; i < kPPRows * upr; i += 256) {
    const int r = i / upr, u = i % upr;
    const int blk = r0 + r;
    float acc[VPU];
#pragma unroll
    for (int c = 0; c < VPU; ++c) acc[c] = 0.0f;
    if (blk < nrows) {
      const int start = blk * b;
      const int cnt = min(b, N - start);
      const uint4* src = reinterpret_cast<const uint4*>(x + (bh * N + start) * d) + u;
      for (int t0 = 0; t0 < cnt; t0 += 8) {
        uint4 buf[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (t0 + j < cnt) buf[j] = __ldg(src + static_cast<long long>(t0 + j) * upr);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (t0 + j < cnt) {
            const T* e = reinterpret_cast<const T*>(&buf[j]);
#pragma unroll
            for (int c = 0; c < VPU; ++c) acc[c] = __fadd_rn(acc[c], static_cast<float>(e[c]));
          }
        }
      }
      const float fc = static_cast<float>(cnt);
#pragma unroll
      for (int c = 0; c < VPU; ++c) acc[c] = __fdiv_rn(acc[c], fc);
    }
#pragma unroll
    for (int c = 0; c < VPU; ++c) xs[r][u * VPU + c] = acc[c];
  }
  __syncthreads();
  // projection: thread = output channel c of rows rh*8 .. rh*8+7
  const int c = tid % kDPad, rh = tid / kDPad;
  if (c >= d) return;
  float out[8];
  if (W == nullptr) {
#pragma unroll
    for (int r = 0; r < 8; ++r) out[r] = xs[rh * 8 + r][c];
  } else {
#pragma unroll
    for (int r = 0; r < 8; ++r) out[r] = 0.0f;
    for (int e = 0; e < d; e += 4) {  // d % 4 == 0
      float w[4];
#pragma unroll
      for (int uu = 0; uu < 4; ++uu) w[uu] = __ldg(W + (e + uu) * d + c);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float4 x4 = *reinterpret_cast<const float4*>(&xs[rh * 8 + r][e]);
        out[r] = __fmaf_rn(x4.x, w[0], out[r]);
        out[r] = __fmaf_rn(x4.y, w[1], out[r]);
        out[r] = __fmaf_rn(x4.z, w[2], out[r]);
        out[r] = __fmaf_rn(x4.w, w[3], out[r]);
      }
    }
  }
  const int stride = isK ? kstride : nrows;  // key rows padded to a multiple of 4 floats
  float* dst = xtT + (bh * d + c) * stride + r0 + rh * 8;
#pragma unroll
  for (int r = 0; r < 8; ++r)
    if (r0 + rh * 8 + r < nrows) dst[r] = out[r];
}

// ---------------------------------------------------------------- scores + selection
// Block: 256 threads, kScoreRows = 8 query blocks of one head.  The scores are
// a small fp32 GEMM: per 256-key pass, thread (ry, kx) forms rows 2ry, 2ry+1 x
// keys 4kx .. 4kx+3 (two shared-memory reads per eight products), the
// projected keys streaming through a double-buffered cp.async ring of
// kScoreC-channel slices.  Every score is a multiply-add chain over c
// ascending, one rounding each.  Then warp w selects for row w.
constexpr int kScoreRows = 8;
constexpr int kScoreKeys = 256;
constexpr int kScoreC = 16;

__global__ void __launch_bounds__(256) score_select_kernel(const float* __restrict__ qtT,
                                                           const float* __restrict__ ktT, int nq, int nkv,
                                                           int kstride, int d, int mode, int k_keep, int k_neg,
                                                           int32_t* __restrict__ kept_idx,
                                                           int8_t* __restrict__ labels,
                                                           float* __restrict__ scores_dbg) {
  extern __shared__ __align__(16) float sm[];
  float* qsT = sm;                              // [128 channels][8 rows]
  float* kbuf = qsT + kDPad * kScoreRows;       // 2 x [kScoreC][kScoreKeys]
  float* sc = kbuf + 2 * kScoreC * kScoreKeys;  // [kScoreRows][nkv]
  const long long bh = blockIdx.y;
  const int r0 = blockIdx.x * kScoreRows;
  const int tid = threadIdx.x;
  for (int i = tid; i < kScoreRows * kDPad; i += 256) {
    const int r = i % kScoreRows, c = i / kScoreRows;
    qsT[i] = (c < d && r0 + r < nq) ? qtT[(bh * d + c) * nq + r0 + r] : 0.0f;
  }
  const float* kbase = ktT + bh * d * static_cast<long long>(kstride);
  const int ry = tid / 64, kx = tid % 64;
  const int nslices = (d + kScoreC - 1) / kScoreC;  // channels past d (d % 16 == 8) are zero-filled
  for (int k0 = 0; k0 < nkv; k0 += kScoreKeys) {
    const int kend = min(kScoreKeys, kstride - k0);  // keys of this pass inside the padded rows
    // slice s of this pass into buffer s & 1: kScoreC rows of kend floats, 16 bytes per copy
    auto load_slice = [&](int sl) {
      float* dstb = kbuf + (sl & 1) * kScoreC * kScoreKeys;
      for (int i = tid; i < kScoreC * (kScoreKeys / 4); i += 256) {
        const int cc = i / (kScoreKeys / 4), k4 = 4 * (i % (kScoreKeys / 4));
        if (sl * kScoreC + cc >= d)
          *reinterpret_cast<float4*>(dstb + cc * kScoreKeys + k4) = make_float4(0.f, 0.f, 0.f, 0.f);
        else if (k4 < kend)
          cp_async16(dstb + cc * kScoreKeys + k4, kbase + static_cast<long long>(sl * kScoreC + cc) * kstride + k0 + k4);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    __syncthreads();  // the previous pass is done with both buffers (and qsT is ready on the first)
    load_slice(0);
    float acc[2][4];
#pragma unroll
    for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
      for (int b4 = 0; b4 < 4; ++b4) acc[a2][b4] = 0.0f;
    for (int sl = 0; sl < nslices; ++sl) {
      if (sl + 1 < nslices) {
        load_slice(sl + 1);
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      }
      __syncthreads();  // slice sl visible to every thread
      const float* kb = kbuf + (sl & 1) * kScoreC * kScoreKeys;
#pragma unroll
      for (int cc = 0; cc < kScoreC; ++cc) {
        const int c = sl * kScoreC + cc;
        const float2 q2 = *reinterpret_cast<const float2*>(qsT + c * kScoreRows + 2 * ry);
        const float4 k4 = *reinterpret_cast<const float4*>(kb + cc * kScoreKeys + 4 * kx);
        const float qa[2] = {q2.x, q2.y};
        const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
          for (int b4 = 0; b4 < 4; ++b4) acc[a2][b4] = __fmaf_rn(qa[a2], kv[b4], acc[a2][b4]);
      }
      __syncthreads();  // buffer sl & 1 may be refilled
    }
#pragma unroll
    for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
      for (int b4 = 0; b4 < 4; ++b4) {
        const int j = k0 + 4 * kx + b4;
        if (j < nkv) sc[(2 * ry + a2) * nkv + j] = acc[a2][b4];
      }
  }
  __syncthreads();

  const int lane = tid % 32, warp = tid / 32;
  {
    const int r = warp;
    const int row = r0 + r;
    if (row >= nq) return;
    const float* srow = sc + r * nkv;
    const long long grow = bh * nq + row;
    // Rank keys: the scores mapped to unsigned integers in the same order
    // (-0 taken as +0, as the comparison does); the k-th largest is found bit
    // by bit with warp-wide counts, ties at it go by block index.
    uint32_t* orow = reinterpret_cast<uint32_t*>(sc + r * nkv);
    for (int j = lane; j < nkv; j += 32) {
      const float sv = srow[j];
      if (scores_dbg) scores_dbg[grow * nkv + j] = sv;
      uint32_t u = __float_as_uint(sv);
      if (u == 0x80000000u) u = 0u;
      orow[j] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    }
    __syncwarp();
    auto count_ge = [&](uint32_t cand, uint32_t flip) -> int {
      int c = 0;
      for (int j = lane; j < nkv; j += 32) c += ((orow[j] ^ flip) >= cand) ? 1 : 0;
      return __reduce_add_sync(0xffffffffu, c);
    };
    // largest T with at least k keys >= T (flip = ~0: keys of the worst blocks)
    auto kth_key = [&](int k, uint32_t flip) -> uint32_t {
      uint32_t T = 0;
      for (int b = 31; b >= 0; --b) {
        const uint32_t cand = T | (1u << b);
        if (count_ge(cand, flip) >= k) T = cand;
      }
      return T;
    };
    const int nt = (nkv + 31) / 32;
    uint64_t top = 0, bot = 0;  // bit t <-> block lane + 32 t
    if (k_keep > 0) {
      // the first k_keep in (score desc, index asc)
      const uint32_t T = kth_key(k_keep, 0u);
      const int need = k_keep - (T == 0xFFFFFFFFu ? 0 : count_ge(T + 1u, 0u));  // from the ties at T
      int seen = 0;
      for (int t = 0; t < nt; ++t) {  // ascending index: the lower indices win the ties
        const int j = lane + 32 * t;
        const uint32_t o = j < nkv ? orow[j] : 0u;
        const bool eq = j < nkv && o == T;
        const uint32_t m = __ballot_sync(0xffffffffu, eq);
        const int rank = seen + __popc(m & ((1u << lane) - 1u));
        if (j < nkv && (o > T || (eq && rank < need))) top |= 1ull << t;
        seen += __popc(m);
      }
    }
    if (mode == SLA_MODE_SLA_3WAY && k_neg > 0) {
      // the last k_neg in (score desc, index asc): lowest scores, higher index first
      const uint32_t T = kth_key(k_neg, 0xFFFFFFFFu);
      const int need = k_neg - (T == 0xFFFFFFFFu ? 0 : count_ge(T + 1u, 0xFFFFFFFFu));
      int seen = 0;
      for (int t = nt - 1; t >= 0; --t) {  // descending index: the higher indices go first
        const int j = lane + 32 * t;
        const uint32_t o = j < nkv ? ~orow[j] : 0u;
        const bool eq = j < nkv && o == T;
        const uint32_t m = __ballot_sync(0xffffffffu, eq);
        const int rank = seen + __popc(m & ~((2u << lane) - 1u));  // equal keys on higher lanes
        if (j < nkv && (o > T || (eq && rank < need))) bot |= 1ull << t;
        seen += __popc(m);
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
      if (j < nkv && labels) labels[grow * nkv + j] = s ? 1 : (((bot >> t) & 1ull) ? -1 : 0);
    }
  }
}

// ---------------------------------------------------------------- launchers

cudaError_t launch_route(const sla_shape& s, const void* q, const void* k, const float* Wq, const float* Wk,
                         int mode, int k_keep, int k_neg, int32_t* kept_idx, int8_t* labels,
                         float* scores_dbg, const WsLayout& L, char* ws, cudaStream_t st) {
  const int BH = s.B * s.H;
  const int nq = ceil_div(s.N, s.bq), nkv = ceil_div(s.N, s.bkv);
  float* qtT = reinterpret_cast<float*>(ws + L.qt);
  float* ktT = reinterpret_cast<float*>(ws + L.kt);
  {
    dim3 grid(ceil_div(nkv > nq ? nkv : nq, kPPRows), BH, 2);
    if (s.in_dtype == SLA_BF16)
      pool_project_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                                                static_cast<const __nv_bfloat16*>(k), Wq, Wk,
                                                                qtT, ktT, s.N, s.d, s.bq, s.bkv, kt_stride(nkv));
    else
      pool_project_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                                        Wq, Wk, qtT, ktT, s.N, s.d, s.bq, s.bkv, kt_stride(nkv));
  }
  {
    const size_t smem =
        (static_cast<size_t>(kDPad) * kScoreRows + 2 * kScoreC * kScoreKeys + static_cast<size_t>(kScoreRows) * nkv) * 4;
    cudaError_t e = cudaFuncSetAttribute(score_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid(ceil_div(nq, kScoreRows), BH);
    score_select_kernel<<<grid, 256, smem, st>>>(qtT, ktT, nq, nkv, kt_stride(nkv), s.d, mode, k_keep, k_neg,
                                                 kept_idx, labels, scores_dbg);
  }
  return cudaGetLastError();
}

}  // namespace sla
