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
                                                           const float* __restrict__ kbar, int N, int d, int bq,
                                                           int bkv, int kstride) {
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
  if (isK && kbar != nullptr) {
    // the key-block means from the prepass (same arithmetic, K read only once)
    for (int i = tid; i < kPPRows * d; i += 256) {
      const int r = i / d, c = i % d;
      xs[r][c] = r0 + r < nrows ? kbar[(bh * nrows + r0 + r) * kDPad + c] : 0.0f;
    }
  } else
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
// Block: 128 threads, kScoreRows = 8 query blocks of one head (three blocks fit
// an SM, so a head-major grid runs in one wave with at most 24 rows per SM).
// The scores are a small fp32 GEMM, taken 512 keys per pass: warp w forms rows
// 4 (w % 2) .. +3 against keys 256 (w / 2) + 4 lane .. +3 and 256 (w / 2) +
// 128 + 4 lane .. +3 of the pass, so each channel costs a thread one broadcast
// read of its four query values and two conflict-free reads of its eight keys
// for 32 products.  The projected keys stream through a kScoreStages-deep
// cp.async ring of kScoreC-channel slices.  Every score is a multiply-add chain
// over c ascending, one rounding each.  Then each warp selects for two rows.
constexpr int kScoreRows = 8;
constexpr int kScoreThreads = 128;
constexpr int kScoreKeys = 512;
constexpr int kScoreC = 8;
constexpr int kScoreStages = 3;

__host__ __device__ constexpr size_t score_smem_bytes(int kstride) {
  return (static_cast<size_t>(kDPad) * kScoreRows + static_cast<size_t>(kScoreStages) * kScoreC * kScoreKeys +
          static_cast<size_t>(kScoreRows) * kstride) * 4;
}

template <int kKPL>  // keys per lane held in registers by the selection: n_kv <= 32 kKPL
__global__ void __launch_bounds__(kScoreThreads) score_select_kernel(const float* __restrict__ qtT,
                                                           const float* __restrict__ ktT, int nq, int nkv,
                                                           int kstride, int d, int mode, int k_keep, int k_neg,
                                                           int32_t* __restrict__ kept_idx,
                                                           int8_t* __restrict__ labels,
                                                           float* __restrict__ scores_dbg, float tau,
                                                           float* __restrict__ soft_mask,
                                                           float* __restrict__ soft_lambda) {
  extern __shared__ __align__(16) float sm[];
  float* qsT = sm;                                         // [128 channels][8 rows]
  float* kbuf = qsT + kDPad * kScoreRows;                  // kScoreStages x [kScoreC][kScoreKeys]
  float* sc = kbuf + kScoreStages * kScoreC * kScoreKeys;  // [kScoreRows][kstride]
  const long long bh = blockIdx.y;
  const int r0 = blockIdx.x * kScoreRows;
  const int tid = threadIdx.x;
  for (int i = tid; i < kScoreRows * kDPad; i += kScoreThreads) {
    const int r = i % kScoreRows, c = i / kScoreRows;
    qsT[i] = (c < d && r0 + r < nq) ? qtT[(bh * d + c) * nq + r0 + r] : 0.0f;
  }
  const float* kbase = ktT + bh * d * static_cast<long long>(kstride);
  const int wq = tid / 32;
  const int rq = wq & 1;                                // rows 4 rq .. 4 rq + 3
  const int kc = 256 * (wq >> 1) + 4 * (tid & 31);      // keys kc .. kc + 3, kc + 128 .. kc + 131 of the pass
  const int nslices = d / kScoreC;                      // d % 8 == 0
  for (int k0 = 0; k0 < nkv; k0 += kScoreKeys) {
    const int kend = min(kScoreKeys, kstride - k0);     // keys of this pass inside the padded rows
    // slice sl (channels kScoreC sl ..) into stage sl % kScoreStages, 16 bytes per copy; a
    // group is committed even when empty so the wait counts stay aligned
    auto load_slice = [&](int sl) {
      if (sl < nslices) {
        float* dstb = kbuf + (sl % kScoreStages) * kScoreC * kScoreKeys;
        for (int i = tid; i < kScoreC * (kScoreKeys / 4); i += kScoreThreads) {
          const int cc = i / (kScoreKeys / 4), k4 = 4 * (i % (kScoreKeys / 4));
          if (k4 < kend)
            cp_async16(dstb + cc * kScoreKeys + k4, kbase + static_cast<long long>(sl * kScoreC + cc) * kstride + k0 + k4);
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    __syncthreads();  // the previous pass is done with every stage (and qsT is ready on the first)
#pragma unroll
    for (int sl = 0; sl < kScoreStages - 1; ++sl) load_slice(sl);
    float acc[4][8];
#pragma unroll
    for (int a4 = 0; a4 < 4; ++a4)
#pragma unroll
      for (int b8 = 0; b8 < 8; ++b8) acc[a4][b8] = 0.0f;
    for (int sl = 0; sl < nslices; ++sl) {
      asm volatile("cp.async.wait_group %0;" ::"n"(kScoreStages - 2) : "memory");
      __syncthreads();  // slice sl visible to every thread; stage (sl - 1) % kScoreStages free again
      load_slice(sl + kScoreStages - 1);
      const float* kb = kbuf + (sl % kScoreStages) * kScoreC * kScoreKeys + kc;
#pragma unroll
      for (int cc = 0; cc < kScoreC; ++cc) {
        const int c = sl * kScoreC + cc;
        const float4 q4 = *reinterpret_cast<const float4*>(qsT + c * kScoreRows + 4 * rq);
        const float4 ka = *reinterpret_cast<const float4*>(kb + cc * kScoreKeys);
        const float4 kb4 = *reinterpret_cast<const float4*>(kb + cc * kScoreKeys + 128);
        const float qa[4] = {q4.x, q4.y, q4.z, q4.w};
        const float kv[8] = {ka.x, ka.y, ka.z, ka.w, kb4.x, kb4.y, kb4.z, kb4.w};
#pragma unroll
        for (int a4 = 0; a4 < 4; ++a4)
#pragma unroll
          for (int b8 = 0; b8 < 8; ++b8) acc[a4][b8] = __fmaf_rn(qa[a4], kv[b8], acc[a4][b8]);
      }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
    for (int a4 = 0; a4 < 4; ++a4)
#pragma unroll
      for (int b8 = 0; b8 < 8; ++b8) {
        const int j = k0 + kc + (b8 & 3) + 128 * (b8 >> 2);
        if (j < nkv) sc[(4 * rq + a4) * kstride + j] = acc[a4][b8];
      }
  }
  __syncthreads();

  const int lane = tid % 32, warp = tid / 32;
  if (soft_mask != nullptr) {
    // SoftTop-k: M = sigmoid(s / tau + lambda), lambda by bisection so that the
    // row's soft selections sum to k_keep (fp32).  The bracket
    // [-max(x) - 40, -min(x) + 40] holds the root; the bisection stops when the
    // midpoint no longer moves.  The row sum of each probe is broadcast from
    // lane 0, so every lane takes the same branch.
    auto sig = [](float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); };  // 0 when e^-z overflows
    for (int r = warp; r < kScoreRows; r += kScoreThreads / 32) {
      const int row = r0 + r;
      if (row >= nq) break;
      const float* srow = sc + r * kstride;
      const long long grow = bh * nq + row;
      const int nvl = nkv > lane ? (nkv - lane + 31) / 32 : 0;
      float x[kKPL];
      float xmax = -INFINITY, xmin = INFINITY;
#pragma unroll
      for (int t = 0; t < kKPL; ++t) {
        x[t] = 0.0f;
        if (t < nvl) {
          const float sv = srow[lane + 32 * t];
          if (scores_dbg) scores_dbg[grow * nkv + lane + 32 * t] = sv;
          x[t] = __fdiv_rn(sv, tau);
          xmax = fmaxf(xmax, x[t]);
          xmin = fminf(xmin, x[t]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        xmax = fmaxf(xmax, __shfl_xor_sync(0xffffffffu, xmax, o));
        xmin = fminf(xmin, __shfl_xor_sync(0xffffffffu, xmin, o));
      }
      float lam = k_keep <= 0 ? -INFINITY : INFINITY;
      if (k_keep > 0 && k_keep < nkv) {
        const float kf = static_cast<float>(k_keep);
        float lo = -xmax - 40.0f, hi = -xmin + 40.0f;
        for (int it = 0; it < 256; ++it) {
          const float mid = 0.5f * (lo + hi);
          if (mid == lo || mid == hi) break;
          float f = 0.0f;
#pragma unroll
          for (int t = 0; t < kKPL; ++t)
            if (t < nvl) f += sig(x[t] + mid);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) f += __shfl_xor_sync(0xffffffffu, f, o);
          f = __shfl_sync(0xffffffffu, f, 0);
          if (f < kf) lo = mid;
          else hi = mid;
        }
        lam = 0.5f * (lo + hi);
      }
#pragma unroll
      for (int t = 0; t < kKPL; ++t) {
        if (t < nvl) {
          const float m = k_keep <= 0 ? 0.0f : (k_keep >= nkv ? 1.0f : sig(x[t] + lam));
          soft_mask[grow * nkv + lane + 32 * t] = m;
        }
      }
      if (lane == 0 && soft_lambda != nullptr) soft_lambda[grow] = lam;
    }
    return;
  }
  for (int r = warp; r < kScoreRows; r += kScoreThreads / 32) {
    const int row = r0 + r;
    if (row >= nq) break;
    const float* srow = sc + r * kstride;
    const long long grow = bh * nq + row;
    // Rank keys: the scores mapped to unsigned integers in the same order
    // (-0 taken as +0, as the comparison does), held in registers: lane l has
    // the keys of blocks l + 32 t, t < nvl.  The k-th largest is found bit by
    // bit with warp-wide counts, ties at it go by block index.
    const int nvl = nkv > lane ? (nkv - lane + 31) / 32 : 0;  // this lane's blocks
    uint32_t key[kKPL];
#pragma unroll
    for (int t = 0; t < kKPL; ++t) {
      const int j = lane + 32 * t;
      uint32_t u = 0u;
      if (t < nvl) {
        const float sv = srow[j];
        if (scores_dbg) scores_dbg[grow * nkv + j] = sv;
        u = __float_as_uint(sv);
        if (u == 0x80000000u) u = 0u;
        u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
      }
      key[t] = u;
    }
    // keys >= cand over the warp: a ballot per register slot (no reduction step)
    auto count_ge = [&](uint32_t cand, uint32_t flip) -> int {
      int c = 0;
#pragma unroll
      for (int t = 0; t < kKPL; ++t) c += __popc(__ballot_sync(0xffffffffu, t < nvl && (key[t] ^ flip) >= cand));
      return c;
    };
    // A threshold T that selects the k best blocks: the largest T with at least
    // k keys >= T (flip = ~0: keys of the worst blocks), found bit by bit.  The
    // search stops early at a candidate with exactly k keys >= it: the keys >= it
    // are then the k largest, and the selection below (keys > T, then keys == T
    // by index up to k) takes exactly those.
    auto kth_key = [&](int k, uint32_t flip) -> uint32_t {
      uint32_t T = 0;
      for (int b = 31; b >= 0; --b) {
        const uint32_t cand = T | (1u << b);
        const int cnt = count_ge(cand, flip);
        if (cnt >= k) T = cand;
        if (cnt == k) break;
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
#pragma unroll
      for (int t = 0; t < kKPL; ++t) {  // ascending index: the lower indices win the ties
        if (t < nt) {
          const bool v = t < nvl;
          const uint32_t o = key[t];
          const bool eq = v && o == T;
          const uint32_t m = __ballot_sync(0xffffffffu, eq);
          const int rank = seen + __popc(m & ((1u << lane) - 1u));
          if (v && (o > T || (eq && rank < need))) top |= 1ull << t;
          seen += __popc(m);
        }
      }
    }
    if (mode == SLA_MODE_SLA_3WAY && k_neg > 0) {
      // the last k_neg in (score desc, index asc): lowest scores, higher index first
      const uint32_t T = kth_key(k_neg, 0xFFFFFFFFu);
      const int need = k_neg - (T == 0xFFFFFFFFu ? 0 : count_ge(T + 1u, 0xFFFFFFFFu));
      int seen = 0;
#pragma unroll
      for (int t = kKPL - 1; t >= 0; --t) {  // descending index: the higher indices go first
        if (t < nt) {
          const bool v = t < nvl;
          const uint32_t o = ~key[t];
          const bool eq = v && o == T;
          const uint32_t m = __ballot_sync(0xffffffffu, eq);
          const int rank = seen + __popc(m & ~((2u << lane) - 1u));  // equal keys on higher lanes
          if (v && (o > T || (eq && rank < need))) bot |= 1ull << t;
          seen += __popc(m);
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
      if (j < nkv && labels) labels[grow * nkv + j] = s ? 1 : (((bot >> t) & 1ull) ? -1 : 0);
    }
  }
}

// ---------------------------------------------------------------- launchers

cudaError_t launch_route(const sla_shape& s, const void* q, const void* k, const float* Wq, const float* Wk,
                         int mode, int k_keep, int k_neg, int32_t* kept_idx, int8_t* labels,
                         float* scores_dbg, const WsLayout& L, char* ws, cudaStream_t st, float tau,
                         float* soft_mask, float* soft_lambda, const float* kbar) {
  const int BH = s.B * s.H;
  const int nq = ceil_div(s.N, s.bq), nkv = ceil_div(s.N, s.bkv);
  float* qtT = reinterpret_cast<float*>(ws + L.qt);
  float* ktT = reinterpret_cast<float*>(ws + L.kt);
  {
    dim3 grid(ceil_div(nkv > nq ? nkv : nq, kPPRows), BH, 2);
    if (s.in_dtype == SLA_BF16)
      pool_project_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                                                static_cast<const __nv_bfloat16*>(k), Wq, Wk,
                                                                qtT, ktT, kbar, s.N, s.d, s.bq, s.bkv,
                                                                kt_stride(nkv));
    else
      pool_project_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                                        Wq, Wk, qtT, ktT, kbar, s.N, s.d, s.bq, s.bkv,
                                                        kt_stride(nkv));
  }
  {
    const size_t smem = score_smem_bytes(kt_stride(nkv));
    const dim3 grid(ceil_div(nq, kScoreRows), BH);
    auto run = [&](auto kernel) -> cudaError_t {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      kernel<<<grid, kScoreThreads, smem, st>>>(qtT, ktT, nq, nkv, kt_stride(nkv), s.d, mode, k_keep, k_neg, kept_idx, labels,
                                      scores_dbg, tau, soft_mask, soft_lambda);
      return cudaSuccess;
    };
    static_assert(kMaxNKV <= 32 * 64, "selection keys per lane");
    const cudaError_t e = nkv <= 512 ? run(score_select_kernel<16>)
                          : nkv <= 1024 ? run(score_select_kernel<32>) : run(score_select_kernel<64>);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace sla
