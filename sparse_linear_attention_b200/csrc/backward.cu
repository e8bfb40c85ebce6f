// backward.cu -- gradients of the SLA2 forward (dQ, dK, dV, d alpha) with the
// block mask held fixed.
//
// Follows "SLA: Beyond Sparsity in Diffusion Transformers …" (papernotes.org)
// 关键设计 4 (the sparse part is back-propagated the FlashAttention way; the
// linear part by the chain rule through dH_i and dZ_i, which are formed per
// query block and aggregated by matrix additions) and "SLA2 深度解读 …"
// (jefxiong.cn) §07 / "SLA2: Sparse-Linear Attention with Learnable Routing
// and QAT" (gist.science) §2.C (gradients on the original, unquantised
// inputs).  The hard Top-k passes no gradient; the router learns through
// SoftTop-k in its own training stage (§06).
//
// Forward being differentiated, per query block i with kept key set S_i and
// the other keys U_i:
//   O   = alpha_i O_s + (1 - alpha_i) O_l
//   O_s = softmax(Q K_S^T / sqrt(d)) V_S
//   O_l = phi(Q) H_i / (phi(Q) . Z_i),  H_i = sum_{m in U_i} phi(k_m)^T v_m,
//                                       Z_i = sum_{m in U_i} phi(k_m)
// The linear branch is written as totals minus the kept blocks, as in the
// forward kernel: H_i = H_tot - sum_{j in S_i} phi(K_j)^T V_j, and the
// gradient that H_i, Z_i send to the keys of U_i as (dH_tot, dZ_tot) minus the
// kept blocks' share.  With A_j = phi(Q) phi(K_j)^T, G_j = dO V_j^T,
// s_r = (1 - alpha) / den_r and dden_r = -(1 - alpha) dO_r . O_l,r / den_r:
//   num        = phi(Q) H_tot - sum_j A_j V_j,  den = phi(Q) . Z_tot - sum_j rowsum(A_j)
//   dS_j       = P_j * (alpha G_j - D),  D_r = alpha dO_r . O_s,r
//   dQ         = dS K / sqrt(d) + phi'(Q) [ s dO H_tot^T + dden Z_tot^T - sum_j Bx_j phi(K_j) ]
//   Bx_j       = s G_j + dden 1^T
//   dK_j      += dS_j^T Q / sqrt(d)               (sparse share)
//   dV_j      += (alpha P_j - s A_j)^T dO         (sparse share minus the kept linear share)
//   dphi(K_j) -= Bx_j^T phi(Q)                    (kept linear share)
//   dH_tot    += phi(Q)^T (s dO),  dZ_tot += phi(Q)^T dden
// and per key, once every query block is done:
//   dphi(k_m) += dH_tot v_m + dZ_tot,  dv_m += dH_tot^T phi(k_m),  dk_m += phi'(k_m) dphi(k_m).
// Every valid key of every head takes that last step, so keys kept by some
// query blocks and not by others get both shares.
//
// Three kernels, all fp32 on the CUDA cores (this is the first, correctness-
// first form; the products are 32x64x128 tiles staged in shared memory):
//   bwd_totals_kernel  H_tot, Z_tot per head (atomic adds over token splits)
//   bwd_query_kernel   one CTA per 32 query rows: three passes over the kept
//                      blocks (row max; row sum, O_s, num, den; gradients)
//   bwd_keys_kernel    the per-key step above
// Key-side gradients are accumulated with fp32 atomic adds, so their rounding
// order (not their value) varies from run to run.
#include <cuda_bf16.h>
#include <math_constants.h>
#include <stdint.h>

#include "sla_device.cuh"
#include "sla_internal.h"
#include "sla_kernels.h"

namespace sla {

namespace {

constexpr int kBT = 256;             // threads per CTA, all three kernels
constexpr int kRowsB = 32;           // query rows per CTA of bwd_query_kernel
constexpr int kLd = kDPad + 4;       // fp32 stride of [token][channel] tiles (16-byte aligned rows)
constexpr int kLdT = kBlockKV + 4;   // fp32 stride of [row][key] tiles
constexpr int kTokTile = 32;         // tokens per staged tile in the totals and keys kernels

__device__ __forceinline__ float ld_in(const float* p) { return *p; }
__device__ __forceinline__ float ld_in(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
// reductions over the 16 lanes of a half warp
__device__ __forceinline__ float half_sum(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float half_max(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Rows [t0, t0 + nrows) of one head's x [N][d] into fp32 tiles with stride kLd:
// xs gets the values (zero past `lim` or past d), ph gets phi of the row (zero
// past d; rows at or past `lim` get zeros when zero_phi_past, else phi of the
// zero vector).  One warp per row, four channels per lane.  Either output may
// be null.
template <typename T>
__device__ void load_rows(const T* __restrict__ x, int lim, int d, int t0, int nrows, float* xs, float* ph,
                          int phi_kind, bool zero_phi_past) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < nrows; r += kBT / 32) {
    const int tok = t0 + r;
    const bool valid = tok < lim;
    float val[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = lane * 4 + u;
      val[u] = (valid && c < d) ? ld_in(x + static_cast<long long>(tok) * d + c) : 0.0f;
    }
    if (xs != nullptr) {
#pragma unroll
      for (int u = 0; u < 4; ++u) xs[r * kLd + lane * 4 + u] = val[u];
    }
    if (ph != nullptr) {
      float f[4];
      if (phi_kind == SLA_PHI_SOFTMAX) {
        float mx = -CUDART_INF_F;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (lane * 4 + u < d) mx = fmaxf(mx, val[u]);
        mx = warp_max(mx);
        float e[4], s = 0.0f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          e[u] = (lane * 4 + u < d) ? expf(val[u] - mx) : 0.0f;
          s += e[u];
        }
        s = warp_sum(s);
#pragma unroll
        for (int u = 0; u < 4; ++u) f[u] = e[u] / s;
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) f[u] = (lane * 4 + u < d) ? (val[u] > 0.0f ? val[u] + 1.0f : expf(val[u])) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) ph[r * kLd + lane * 4 + u] = (!valid && zero_phi_past) ? 0.0f : f[u];
    }
  }
}

// dL/dx for one row held four channels per lane across a warp (phi' of the
// feature map; the softmax needs the row sum of dphi * phi).
__device__ __forceinline__ void phi_grad_row(int phi_kind, const float x[4], const float f[4], const float g[4],
                                             float out[4]) {
  if (phi_kind == SLA_PHI_SOFTMAX) {
    const float dot = warp_sum(g[0] * f[0] + g[1] * f[1] + g[2] * f[2] + g[3] * f[3]);
#pragma unroll
    for (int u = 0; u < 4; ++u) out[u] = f[u] * (g[u] - dot);
  } else {
#pragma unroll
    for (int u = 0; u < 4; ++u) out[u] = g[u] * (x[u] > 0.0f ? 1.0f : expf(x[u]));
  }
}

// ---------------------------------------------------------------- totals
// grid (splits, BH): H_tot[e][c] += sum_n phi(k_n)[e] v_n[c], Z_tot[e] += sum_n phi(k_n)[e]
// over the split's tokens.  Thread: row e = tid / 2, columns 64 (tid % 2) .. +63.
template <typename T>
__global__ void __launch_bounds__(kBT) bwd_totals_kernel(const T* __restrict__ k, const T* __restrict__ v, int N,
                                                         int d, int phi_kind, int tok_per_split,
                                                         float* __restrict__ Htot, float* __restrict__ Ztot) {
  extern __shared__ __align__(16) float smb[];
  float* phk = smb;                 // [32][kLd]
  float* vs = smb + kTokTile * kLd;  // [32][kLd]
  const long long bh = blockIdx.y;
  const int t_begin = blockIdx.x * tok_per_split;
  const int t_end = min(N, t_begin + tok_per_split);
  if (t_begin >= t_end) return;
  const T* kb = k + bh * N * d;
  const T* vb = v + bh * N * d;
  const int tid = threadIdx.x, e = tid >> 1, c0 = (tid & 1) * 64;
  float h[64];
#pragma unroll
  for (int u = 0; u < 64; ++u) h[u] = 0.0f;
  float z = 0.0f;
  for (int t0 = t_begin; t0 < t_end; t0 += kTokTile) {
    __syncthreads();
    load_rows(kb, t_end, d, t0, kTokTile, nullptr, phk, phi_kind, true);
    load_rows(vb, t_end, d, t0, kTokTile, vs, nullptr, phi_kind, true);
    __syncthreads();
    const int nt = min(kTokTile, t_end - t0);
    for (int t = 0; t < nt; ++t) {
      const float pe = phk[t * kLd + e];
      const float4* vr = reinterpret_cast<const float4*>(vs + t * kLd + c0);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float4 w = vr[u];
        h[4 * u] = fmaf(pe, w.x, h[4 * u]);
        h[4 * u + 1] = fmaf(pe, w.y, h[4 * u + 1]);
        h[4 * u + 2] = fmaf(pe, w.z, h[4 * u + 2]);
        h[4 * u + 3] = fmaf(pe, w.w, h[4 * u + 3]);
      }
      z += pe;
    }
  }
  if (e < d) {
    float* hrow = Htot + (bh * kDPad + e) * kDPad + c0;
#pragma unroll
    for (int u = 0; u < 64; ++u)
      if (c0 + u < d) atomicAdd(hrow + u, h[u]);
    if ((tid & 1) == 0) atomicAdd(Ztot + bh * kDPad + e, z);
  }
}

// ---------------------------------------------------------------- per query tile
struct BwdArgs {
  const void *q, *k, *v, *dout;
  const int32_t* kept;
  const float* alpha;
  int N, d, bq, nq, nkv, kk, phi;
  float scale;
  const float *Htot, *Ztot;
  float *dHtot, *dZtot, *dphik;
  float *dq, *dk, *dv, *dalpha;
  int* status;
  // SLA (sla != 0): per query block the critical and negligible lists
  // [rows][2][nkv] with their counts [rows][2], W_proj [d][d], and the O_l
  // rows [BH][N][128] kept for dW_proj.  kept, kk, alpha and dalpha unused.
  int sla;
  const int32_t *lists, *counts;
  const __nv_bfloat16* wproj;
  float* ol;
};

// Shared-memory layout of bwd_query_kernel (floats)
constexpr int kOffQ = 0;
constexpr int kOffPQ = kOffQ + kRowsB * kLd;
constexpr int kOffDO = kOffPQ + kRowsB * kLd;
constexpr int kOffK = kOffDO + kRowsB * kLd;      // K_j [64][kLd]; H_tot staging [128][kLd] before the passes
constexpr int kOffPK = kOffK + kBlockKV * kLd;
constexpr int kOffV = kOffPK + kBlockKV * kLd;
constexpr int kOffT1 = kOffV + kBlockKV * kLd;    // S -> P -> dS  [32][kLdT]
constexpr int kOffT2 = kOffT1 + kRowsB * kLdT;    // A -> C
constexpr int kOffT3 = kOffT2 + kRowsB * kLdT;    // G -> Bx
constexpr int kOffRV = kOffT3 + kRowsB * kLdT;    // row scalars: m, l, rsA, D, s, dden  [6][32]
constexpr int kOffZ = kOffRV + 6 * kRowsB;        // Z_tot [128]
constexpr int kOffRed = kOffZ + kDPad;            // [8] block reduction
constexpr int kOffE = kOffRed + 8;                // SLA: dO_l = dO W_proj^T  [32][kLd]
constexpr int kOffT4 = kOffE + kRowsB * kLd;      // SLA: -s A  [32][kLdT]
constexpr int kQuerySmemFloats = kOffT4 + kRowsB * kLdT;
static_assert(3 * kBlockKV * kLd >= kDPad * kLd, "H_tot staging fits the key tiles");
static_assert(kQuerySmemFloats * 4 <= 232448, "shared memory budget");

// A 32 x 64 product over the channels: out[u2][w] = sum_e X[r][e] Y[c][e] for
// rows r = 2 (tid / 16) + u2 and keys c = tid % 16 + 16 w.
__device__ __forceinline__ void rows_x_keys_over_channels(const float* X, const float* Y, int d, float out[2][4]) {
  const int rg = threadIdx.x >> 4, kl = threadIdx.x & 15;
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int w = 0; w < 4; ++w) out[u][w] = 0.0f;
  for (int e = 0; e < d; e += 4) {
    float4 x[2], y[4];
#pragma unroll
    for (int u = 0; u < 2; ++u) x[u] = *reinterpret_cast<const float4*>(X + (2 * rg + u) * kLd + e);
#pragma unroll
    for (int w = 0; w < 4; ++w) y[w] = *reinterpret_cast<const float4*>(Y + (kl + 16 * w) * kLd + e);
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        out[u][w] = fmaf(x[u].x, y[w].x, out[u][w]);
        out[u][w] = fmaf(x[u].y, y[w].y, out[u][w]);
        out[u][w] = fmaf(x[u].z, y[w].z, out[u][w]);
        out[u][w] = fmaf(x[u].w, y[w].w, out[u][w]);
      }
  }
}

// acc[u][w] += sign * sum_c T[rr][c] Y[c][cc + w] over the 64 keys, for rows
// rr = 4 (tid / 32) + u and channels cc = 4 (tid % 32).
__device__ __forceinline__ void rows_x_channels_over_keys(const float* Tt, const float* Y, float sign,
                                                          float acc[4][4]) {
  const int wr = threadIdx.x >> 5, cc = (threadIdx.x & 31) * 4;
  for (int c = 0; c < kBlockKV; ++c) {
    const float4 y = *reinterpret_cast<const float4*>(Y + c * kLd + cc);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float t = sign * Tt[(4 * wr + u) * kLdT + c];
      acc[u][0] = fmaf(t, y.x, acc[u][0]);
      acc[u][1] = fmaf(t, y.y, acc[u][1]);
      acc[u][2] = fmaf(t, y.z, acc[u][2]);
      acc[u][3] = fmaf(t, y.w, acc[u][3]);
    }
  }
}

// out[u8][w] = sum_r T[r][kr] X[r][cc + w] over the 32 rows, for keys
// kr = 8 (tid / 32) + u8 and channels cc = 4 (tid % 32).
__device__ __forceinline__ void keys_x_channels_over_rows(const float* Tt, const float* X, float out[8][4]) {
  const int wr = threadIdx.x >> 5, cc = (threadIdx.x & 31) * 4;
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int w = 0; w < 4; ++w) out[u][w] = 0.0f;
  for (int r = 0; r < kRowsB; ++r) {
    const float4 x = *reinterpret_cast<const float4*>(X + r * kLd + cc);
    const float4 t0 = *reinterpret_cast<const float4*>(Tt + r * kLdT + 8 * wr);
    const float4 t1 = *reinterpret_cast<const float4*>(Tt + r * kLdT + 8 * wr + 4);
    const float t[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      out[u][0] = fmaf(t[u], x.x, out[u][0]);
      out[u][1] = fmaf(t[u], x.y, out[u][1]);
      out[u][2] = fmaf(t[u], x.z, out[u][2]);
      out[u][3] = fmaf(t[u], x.w, out[u][3]);
    }
  }
}

// Atomic add of a 64 x 128 key-side tile (rows kr = 8 (tid / 32) + u8) into
// dst [N][ld] of one head, keys j * 64 + kr < N and channels < d only.
__device__ __forceinline__ void add_key_tile(float* dst, int ld, int N, int d, int key0, float scale,
                                             const float val[8][4]) {
  const int wr = threadIdx.x >> 5, cc = (threadIdx.x & 31) * 4;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int tok = key0 + 8 * wr + u;
    if (tok < N) {
#pragma unroll
      for (int w = 0; w < 4; ++w)
        if (cc + w < d) atomicAdd(dst + static_cast<long long>(tok) * ld + cc + w, scale * val[u][w]);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kBT, 1) bwd_query_kernel(const BwdArgs a) {
  extern __shared__ __align__(16) float smq[];
  float* Qs = smq + kOffQ;
  float* PQ = smq + kOffPQ;
  float* DO = smq + kOffDO;
  float* Ks = smq + kOffK;
  float* PK = smq + kOffPK;
  float* Vs = smq + kOffV;
  float* T1 = smq + kOffT1;
  float* T2 = smq + kOffT2;
  float* T3 = smq + kOffT3;
  float* rv_m = smq + kOffRV;
  float* rv_l = rv_m + kRowsB;
  float* rv_rsA = rv_l + kRowsB;
  float* rv_D = rv_rsA + kRowsB;
  float* rv_s = rv_D + kRowsB;
  float* rv_dd = rv_s + kRowsB;
  float* Zs = smq + kOffZ;
  float* red = smq + kOffRed;
  float* Es = smq + kOffE;
  float* T4 = smq + kOffT4;

  const int tid = threadIdx.x, lane = tid & 31, wr = tid >> 5;
  const int rg = tid >> 4, kl = tid & 15;  // 32 x 64 tile map
  const int cc = lane * 4;                  // channel columns of the 32 x 128 and 64 x 128 maps
  const int nsub = a.bq / kRowsB;
  const int i = blockIdx.x / nsub;
  const int row0 = i * a.bq + (blockIdx.x % nsub) * kRowsB;
  if (row0 >= a.N) return;
  const long long bh = blockIdx.y;
  const int N = a.N, d = a.d;
  const T* qb = static_cast<const T*>(a.q) + bh * N * d;
  const T* kb = static_cast<const T*>(a.k) + bh * N * d;
  const T* vb = static_cast<const T*>(a.v) + bh * N * d;
  const T* gb = static_cast<const T*>(a.dout) + bh * N * d;
  const long long rowq = bh * a.nq + i;
  // The blocks whose linear share is taken out of the totals: SLA2 the kept
  // list; SLA the critical list, then the negligible one.  The first n_crit
  // of them also take the sparse branch.
  const int32_t* clist;
  const int32_t* nlist = nullptr;
  int n_crit, n_all;
  if (a.sla) {
    clist = a.lists + rowq * 2 * a.nkv;
    nlist = clist + a.nkv;
    n_crit = a.counts[2 * rowq];
    n_all = n_crit + a.counts[2 * rowq + 1];
  } else {
    clist = a.kept + rowq * a.kk;
    n_crit = n_all = a.kk;
  }
  auto entry = [&](int jj) { return jj < n_crit ? clist[jj] : nlist[jj - n_crit]; };
  // dO_s = c_s dO; dO_l = c_l dO (SLA2) or dO W_proj^T (SLA, held in Es)
  const float alpha = a.sla ? 1.0f : a.alpha[rowq];
  const float lin_w = a.sla ? 1.0f : 1.0f - alpha;
  const bool has_lin = n_all < a.nkv;
  const float* LD = a.sla ? Es : DO;
  auto block_ok = [&](int j) { return j >= 0 && j < a.nkv; };

  // rows, phi(rows) (phi of the zero vector past N keeps den > 0), dO, Z_tot, H_tot
  load_rows(qb, N, d, row0, kRowsB, Qs, PQ, a.phi, false);
  load_rows(gb, N, d, row0, kRowsB, DO, nullptr, a.phi, false);
  if (a.sla) {
    // W_proj^T staged [c][e], then E = dO W_proj^T (32 x 128 map)
    for (int x = tid; x < kDPad * kDPad; x += kBT) {
      const int e = x / kDPad, c = x % kDPad;
      Ks[c * kLd + e] = (e < d && c < d) ? __bfloat162float(a.wproj[e * d + c]) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      const int r = 4 * wr + u;
      for (int c = 0; c < d; ++c) {
        const float g = DO[r * kLd + c];
        const float4 wv = *reinterpret_cast<const float4*>(Ks + c * kLd + cc);
        acc[0] = fmaf(g, wv.x, acc[0]);
        acc[1] = fmaf(g, wv.y, acc[1]);
        acc[2] = fmaf(g, wv.z, acc[2]);
        acc[3] = fmaf(g, wv.w, acc[3]);
      }
#pragma unroll
      for (int w = 0; w < 4; ++w) Es[r * kLd + cc + w] = acc[w];
    }
    __syncthreads();
  }
  const float* Hg = a.Htot + bh * kDPad * kDPad;
  for (int x = tid; x < kDPad * kDPad; x += kBT) Ks[(x / kDPad) * kLd + x % kDPad] = Hg[x];
  for (int x = tid; x < kDPad; x += kBT) Zs[x] = a.Ztot[bh * kDPad + x];
  __syncthreads();
  // num = phi(Q) H_tot (32 x 128 map)
  float num[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int w = 0; w < 4; ++w) num[u][w] = 0.0f;
  for (int e = 0; e < d; ++e) {
    const float4 h = *reinterpret_cast<const float4*>(Ks + e * kLd + cc);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float p = PQ[(4 * wr + u) * kLd + e];
      num[u][0] = fmaf(p, h.x, num[u][0]);
      num[u][1] = fmaf(p, h.y, num[u][1]);
      num[u][2] = fmaf(p, h.z, num[u][2]);
      num[u][3] = fmaf(p, h.w, num[u][3]);
    }
  }
  __syncthreads();
  // H_tot^T staged, then hdo = dO H_tot^T
  for (int x = tid; x < kDPad * kDPad; x += kBT) Ks[(x % kDPad) * kLd + x / kDPad] = Hg[x];
  __syncthreads();
  float hdo[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int w = 0; w < 4; ++w) hdo[u][w] = 0.0f;
  for (int c = 0; c < d; ++c) {
    const float4 h = *reinterpret_cast<const float4*>(Ks + c * kLd + cc);  // H_tot[cc + w][c]
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float g = LD[(4 * wr + u) * kLd + c];
      hdo[u][0] = fmaf(g, h.x, hdo[u][0]);
      hdo[u][1] = fmaf(g, h.y, hdo[u][1]);
      hdo[u][2] = fmaf(g, h.z, hdo[u][2]);
      hdo[u][3] = fmaf(g, h.w, hdo[u][3]);
    }
  }

  // ------------------------------------------------ pass 0: row max of the scaled scores
  float m2[2] = {-CUDART_INF_F, -CUDART_INF_F};
  for (int jj = 0; jj < n_crit; ++jj) {
    const int j = entry(jj);
    if (!block_ok(j)) {
      if (tid == 0) report_error(a.status, SLA_ERR_DEVICE_INDEX);
      continue;
    }
    __syncthreads();
    load_rows(kb, N, d, j * kBlockKV, kBlockKV, Ks, nullptr, a.phi, true);
    __syncthreads();
    const int nvalid = min(kBlockKV, N - j * kBlockKV);
    float s[2][4];
    rows_x_keys_over_channels(Qs, Ks, d, s);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float mx = -CUDART_INF_F;
#pragma unroll
      for (int w = 0; w < 4; ++w)
        if (kl + 16 * w < nvalid) mx = fmaxf(mx, s[u][w] * a.scale);
      m2[u] = fmaxf(m2[u], half_max(mx));
    }
  }

  // ------------------------------------------------ pass 1: l, O_s, num, den
  float l2[2] = {0.0f, 0.0f}, rsa2[2] = {0.0f, 0.0f};
  float oacc[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int w = 0; w < 4; ++w) oacc[u][w] = 0.0f;
  for (int jj = 0; jj < n_all; ++jj) {
    const int j = entry(jj);
    if (!block_ok(j)) {
      if (jj >= n_crit && tid == 0) report_error(a.status, SLA_ERR_DEVICE_INDEX);
      continue;
    }
    const bool crit = jj < n_crit;
    __syncthreads();
    load_rows(kb, N, d, j * kBlockKV, kBlockKV, Ks, PK, a.phi, true);
    load_rows(vb, N, d, j * kBlockKV, kBlockKV, Vs, nullptr, a.phi, true);
    __syncthreads();
    const int nvalid = min(kBlockKV, N - j * kBlockKV);
    float s[2][4], al[2][4];
    if (crit) rows_x_keys_over_channels(Qs, Ks, d, s);
    rows_x_keys_over_channels(PQ, PK, d, al);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float ls = 0.0f, as = 0.0f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int c = kl + 16 * w;
        const float p = (crit && c < nvalid) ? expf(s[u][w] * a.scale - m2[u]) : 0.0f;
        T1[(2 * rg + u) * kLdT + c] = p;
        T2[(2 * rg + u) * kLdT + c] = al[u][w];  // phi(K) rows past N are zero
        ls += p;
        as += al[u][w];
      }
      l2[u] += half_sum(ls);
      rsa2[u] += half_sum(as);
    }
    __syncthreads();
    if (crit) rows_x_channels_over_keys(T1, Vs, 1.0f, oacc);
    rows_x_channels_over_keys(T2, Vs, -1.0f, num);
  }
  if (kl == 0) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      rv_m[2 * rg + u] = m2[u];
      rv_l[2 * rg + u] = l2[u];
      rv_rsA[2 * rg + u] = rsa2[u];
    }
  }
  __syncthreads();
  // row scalars in the 32 x 128 map (rows 4 wr + u)
  float dal = 0.0f;
  float sr4[4], dd4[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int r = 4 * wr + u;
    const float l = rv_l[r];
    float os[4], ol[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) os[w] = l > 0.0f ? oacc[u][w] / l : 0.0f;
    float den = 0.0f;
    if (has_lin) {
#pragma unroll
      for (int w = 0; w < 4; ++w) den = fmaf(PQ[r * kLd + cc + w], Zs[cc + w], den);
      den = warp_sum(den) - rv_rsA[r];
    }
#pragma unroll
    for (int w = 0; w < 4; ++w) ol[w] = has_lin ? num[u][w] / den : 0.0f;
    float dos = 0.0f, dol = 0.0f, dlo = 0.0f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float g = DO[r * kLd + cc + w];
      dos = fmaf(g, os[w], dos);
      dol = fmaf(g, ol[w], dol);
      dlo = fmaf(LD[r * kLd + cc + w], ol[w], dlo);
    }
    dos = warp_sum(dos);
    dol = warp_sum(dol);
    dlo = warp_sum(dlo);
    dal += dos - dol;
    // SLA2: s = (1 - alpha) / den with dO; SLA: s = 1 / den with dO W_proj^T
    sr4[u] = has_lin ? lin_w / den : 0.0f;
    dd4[u] = has_lin ? -lin_w * dlo / den : 0.0f;
    if (a.sla && row0 + r < N) {
      float* olr = a.ol + (bh * N + row0 + r) * kDPad + cc;
      *reinterpret_cast<float4*>(olr) = make_float4(ol[0], ol[1], ol[2], ol[3]);
    }
    if (lane == 0) {
      rv_D[r] = alpha * dos;
      rv_s[r] = sr4[u];
      rv_dd[r] = dd4[u];
    }
  }
  if (lane == 0) red[wr] = dal;
  __syncthreads();
  if (tid == 0 && !a.sla) {
    float t = 0.0f;
    for (int w = 0; w < kBT / 32; ++w) t += red[w];
    atomicAdd(a.dalpha + rowq, t);
  }

  // ------------------------------------------------ pass 2: gradients
  float dqa[4][4], dpq[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      dqa[u][w] = 0.0f;
      dpq[u][w] = 0.0f;
    }
  float* dkh = a.dk + bh * N * d;
  float* dvh = a.dv + bh * N * d;
  float* dpkh = a.dphik + bh * N * kDPad;
  for (int jj = 0; jj < n_all; ++jj) {
    const int j = entry(jj);
    if (!block_ok(j)) continue;
    const bool crit = jj < n_crit;
    __syncthreads();
    load_rows(kb, N, d, j * kBlockKV, kBlockKV, Ks, PK, a.phi, true);
    load_rows(vb, N, d, j * kBlockKV, kBlockKV, Vs, nullptr, a.phi, true);
    __syncthreads();
    const int nvalid = min(kBlockKV, N - j * kBlockKV);
    {
      float s[2][4], al[2][4], g[2][4], gl[2][4];
      if (crit) {
        rows_x_keys_over_channels(Qs, Ks, d, s);
        rows_x_keys_over_channels(DO, Vs, d, g);
      }
      rows_x_keys_over_channels(PQ, PK, d, al);
      if (a.sla) rows_x_keys_over_channels(Es, Vs, d, gl);  // SLA2: dO_l V^T = (1 - alpha) G
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int r = 2 * rg + u;
        const float m = rv_m[r], l = rv_l[r], D = rv_D[r], sr = rv_s[r], dd = rv_dd[r];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int c = kl + 16 * w;
          const bool kv = c < nvalid;
          const float p = (crit && kv) ? expf(s[u][w] * a.scale - m) / l : 0.0f;
          const float gs = crit ? g[u][w] : 0.0f;
          const float glv = a.sla ? gl[u][w] : gs;
          T1[r * kLdT + c] = p * (alpha * gs - D);                  // dS
          T2[r * kLdT + c] = a.sla ? p : alpha * p - sr * al[u][w];  // C (SLA: P)
          T3[r * kLdT + c] = kv ? sr * glv + dd : 0.0f;             // Bx
          if (a.sla) T4[r * kLdT + c] = -sr * al[u][w];
        }
      }
    }
    __syncthreads();
    if (crit) rows_x_channels_over_keys(T1, Ks, 1.0f, dqa);
    rows_x_channels_over_keys(T3, PK, -1.0f, dpq);
    {
      float kt[8][4];
      if (crit) {
        keys_x_channels_over_rows(T1, Qs, kt);
        add_key_tile(dkh, d, N, d, j * kBlockKV, a.scale, kt);
      }
      if (a.sla) {
        // dV = P^T dO (critical) - (s A)^T dO_l
        keys_x_channels_over_rows(T4, Es, kt);
        if (crit) {
          float kp[8][4];
          keys_x_channels_over_rows(T2, DO, kp);
#pragma unroll
          for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) kt[u][w] += kp[u][w];
        }
      } else {
        keys_x_channels_over_rows(T2, DO, kt);
      }
      add_key_tile(dvh, d, N, d, j * kBlockKV, 1.0f, kt);
      if (has_lin) {
        keys_x_channels_over_rows(T3, PQ, kt);
        add_key_tile(dpkh, kDPad, N, d, j * kBlockKV, -1.0f, kt);
      }
    }
  }

  // dq of the valid rows
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int r = 4 * wr + u;
    float x[4], f[4], gphi[4], out[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      x[w] = Qs[r * kLd + cc + w];
      f[w] = PQ[r * kLd + cc + w];
      gphi[w] = (cc + w < d) ? dpq[u][w] + sr4[u] * hdo[u][w] + dd4[u] * Zs[cc + w] : 0.0f;
    }
    phi_grad_row(a.phi, x, f, gphi, out);
    const int tok = row0 + r;
    if (tok < N) {
#pragma unroll
      for (int w = 0; w < 4; ++w)
        if (cc + w < d) a.dq[(bh * N + tok) * d + cc + w] = a.scale * dqa[u][w] + out[w];
    }
  }

  // dH_tot += phi(Q)^T (s dO), dZ_tot += phi(Q)^T dden
  if (has_lin) {
    const int e = tid >> 1, c0 = (tid & 1) * 64;
    if (e < d) {
      float h[64];
#pragma unroll
      for (int u = 0; u < 64; ++u) h[u] = 0.0f;
      float z = 0.0f;
      for (int r = 0; r < kRowsB; ++r) {
        const float pe = PQ[r * kLd + e];
        const float ps = pe * rv_s[r];
        const float4* gr = reinterpret_cast<const float4*>(LD + r * kLd + c0);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float4 g = gr[u];
          h[4 * u] = fmaf(ps, g.x, h[4 * u]);
          h[4 * u + 1] = fmaf(ps, g.y, h[4 * u + 1]);
          h[4 * u + 2] = fmaf(ps, g.z, h[4 * u + 2]);
          h[4 * u + 3] = fmaf(ps, g.w, h[4 * u + 3]);
        }
        z = fmaf(pe, rv_dd[r], z);
      }
      float* hrow = a.dHtot + (bh * kDPad + e) * kDPad + c0;
#pragma unroll
      for (int u = 0; u < 64; ++u)
        if (c0 + u < d) atomicAdd(hrow + u, h[u]);
      if ((tid & 1) == 0) atomicAdd(a.dZtot + bh * kDPad + e, z);
    }
  }
}

// ---------------------------------------------------------------- per key
// grid (ceil(N / 32), BH): dphi(k) = (kept shares) + dH_tot v + dZ_tot,
// dv += dH_tot^T phi(k), dk += phi'(k) dphi(k).  32 x 128 map: tokens
// 4 (tid / 32) + u, channels 4 (tid % 32) + w.
constexpr int kKeysSmemFloats = 2 * kDPad * kLd + kDPad + 3 * kTokTile * kLd;
static_assert(kKeysSmemFloats * 4 <= 232448, "shared memory budget");

template <typename T>
__global__ void __launch_bounds__(kBT, 1) bwd_keys_kernel(const T* __restrict__ k, const T* __restrict__ v, int N,
                                                          int d, int phi_kind, const float* __restrict__ dHtot,
                                                          const float* __restrict__ dZtot,
                                                          const float* __restrict__ dphik, float* __restrict__ dk,
                                                          float* __restrict__ dv) {
  extern __shared__ __align__(16) float smk[];
  float* dH = smk;                  // [e][c]
  float* dHT = dH + kDPad * kLd;    // [c][e]
  float* dZ = dHT + kDPad * kLd;
  float* Kt = dZ + kDPad;           // raw k [32][kLd]
  float* PKt = Kt + kTokTile * kLd;  // phi(k)
  float* Vt = PKt + kTokTile * kLd;
  const long long bh = blockIdx.y;
  const int t0 = blockIdx.x * kTokTile;
  if (t0 >= N) return;
  const int tid = threadIdx.x, wr = tid >> 5, cc = (tid & 31) * 4;
  const float* dHg = dHtot + bh * kDPad * kDPad;
  for (int x = tid; x < kDPad * kDPad; x += kBT) {
    const float h = dHg[x];
    dH[(x / kDPad) * kLd + x % kDPad] = h;
    dHT[(x % kDPad) * kLd + x / kDPad] = h;
  }
  for (int x = tid; x < kDPad; x += kBT) dZ[x] = dZtot[bh * kDPad + x];
  load_rows(k + bh * N * d, N, d, t0, kTokTile, Kt, PKt, phi_kind, true);
  load_rows(v + bh * N * d, N, d, t0, kTokTile, Vt, nullptr, phi_kind, true);
  __syncthreads();
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int r = 4 * wr + u;
    const int tok = t0 + r;
    float dvl[4] = {0.0f, 0.0f, 0.0f, 0.0f}, gp[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int e = 0; e < d; ++e) {
      const float pe = PKt[r * kLd + e];
      const float ve = Vt[r * kLd + e];
      const float4 h = *reinterpret_cast<const float4*>(dH + e * kLd + cc);    // dH[e][cc + w]
      const float4 ht = *reinterpret_cast<const float4*>(dHT + e * kLd + cc);  // dH[cc + w][e]
      dvl[0] = fmaf(pe, h.x, dvl[0]);
      dvl[1] = fmaf(pe, h.y, dvl[1]);
      dvl[2] = fmaf(pe, h.z, dvl[2]);
      dvl[3] = fmaf(pe, h.w, dvl[3]);
      gp[0] = fmaf(ve, ht.x, gp[0]);
      gp[1] = fmaf(ve, ht.y, gp[1]);
      gp[2] = fmaf(ve, ht.z, gp[2]);
      gp[3] = fmaf(ve, ht.w, gp[3]);
    }
    float x[4], f[4], out[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      x[w] = Kt[r * kLd + cc + w];
      f[w] = PKt[r * kLd + cc + w];
      const bool ok = tok < N && cc + w < d;
      gp[w] = ok ? gp[w] + dZ[cc + w] + dphik[(bh * N + tok) * kDPad + cc + w] : 0.0f;
    }
    phi_grad_row(phi_kind, x, f, gp, out);
    if (tok < N) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        if (cc + w < d) {
          const long long o = (bh * N + tok) * d + cc + w;
          dk[o] += out[w];
          dv[o] += dvl[w];
        }
      }
    }
  }
}

// ---------------------------------------------------------------- dW_proj (SLA)
// grid (nsplit): this split's share of dW_proj[e][c] = sum over the rows of
// every head of O_l[e] dO[c], rows [split * per, ...) of the flat [BH * N]
// row range; thread: e = tid / 2, columns 64 (tid % 2) .. +63.  The partials
// are summed in split order by bwd_wproj_sum_kernel, so dW_proj is the same
// on every run.
template <typename T>
__global__ void __launch_bounds__(kBT) bwd_wproj_kernel(const float* __restrict__ ol, const T* __restrict__ dout,
                                                        long long rows, int d, long long per,
                                                        float* __restrict__ wpart) {
  extern __shared__ __align__(16) float smw[];
  float* Ot = smw;                   // [32][kLd]
  float* Gt = smw + kTokTile * kLd;  // [32][kLd]
  const long long r_begin = blockIdx.x * per;
  const long long r_end = min(rows, r_begin + per);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, e = tid >> 1, c0 = (tid & 1) * 64;
  float h[64];
#pragma unroll
  for (int u = 0; u < 64; ++u) h[u] = 0.0f;
  for (long long t0 = r_begin; t0 < r_end; t0 += kTokTile) {
    __syncthreads();
    for (int r = warp; r < kTokTile; r += kBT / 32) {
      const long long row = t0 + r;
      const bool valid = row < r_end;
      float4 o = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (valid) o = *reinterpret_cast<const float4*>(ol + row * kDPad + 4 * lane);
      *reinterpret_cast<float4*>(Ot + r * kLd + 4 * lane) = o;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = 4 * lane + u;
        Gt[r * kLd + c] = (valid && c < d) ? ld_in(dout + row * d + c) : 0.0f;
      }
    }
    __syncthreads();
    const int nt = static_cast<int>(min(static_cast<long long>(kTokTile), r_end - t0));
    for (int t = 0; t < nt; ++t) {
      const float oe = Ot[t * kLd + e];
      const float4* gr = reinterpret_cast<const float4*>(Gt + t * kLd + c0);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float4 g = gr[u];
        h[4 * u] = fmaf(oe, g.x, h[4 * u]);
        h[4 * u + 1] = fmaf(oe, g.y, h[4 * u + 1]);
        h[4 * u + 2] = fmaf(oe, g.z, h[4 * u + 2]);
        h[4 * u + 3] = fmaf(oe, g.w, h[4 * u + 3]);
      }
    }
  }
  float* dst = wpart + (static_cast<long long>(blockIdx.x) * kDPad + e) * kDPad + c0;
#pragma unroll
  for (int u = 0; u < 64; u += 4)
    *reinterpret_cast<float4*>(dst + u) = make_float4(h[u], h[u + 1], h[u + 2], h[u + 3]);
}

// dW_proj [d][d] = the partials summed in split order.
__global__ void __launch_bounds__(kBT) bwd_wproj_sum_kernel(const float* __restrict__ wpart, int nsplit, int d,
                                                            float* __restrict__ dwproj) {
  const int x = blockIdx.x * kBT + threadIdx.x;
  if (x >= d * d) return;
  const int e = x / d, c = x % d;
  float t = 0.0f;
  for (int sp = 0; sp < nsplit; ++sp) t += wpart[(static_cast<long long>(sp) * kDPad + e) * kDPad + c];
  dwproj[x] = t;
}

template <typename T>
cudaError_t run_backward(const sla_shape& s, const BwdArgs& a, cudaStream_t st) {
  const int BH = s.B * s.H;
  {
    // token splits: about two CTAs per SM in all
    int splits = (2 * kNumSMs + BH - 1) / BH;
    const int max_splits = (s.N + kTokTile - 1) / kTokTile;
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
    int per = (s.N + splits - 1) / splits;
    per = (per + kTokTile - 1) / kTokTile * kTokTile;
    splits = (s.N + per - 1) / per;
    const size_t smem = 2 * kTokTile * kLd * sizeof(float);
    bwd_totals_kernel<T><<<dim3(splits, BH), kBT, smem, st>>>(static_cast<const T*>(a.k), static_cast<const T*>(a.v),
                                                              s.N, s.d, a.phi, per, const_cast<float*>(a.Htot),
                                                              const_cast<float*>(a.Ztot));
  }
  {
    const size_t smem = kQuerySmemFloats * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(bwd_query_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    bwd_query_kernel<T><<<dim3(a.nq * (s.bq / kRowsB), BH), kBT, smem, st>>>(a);
  }
  {
    const size_t smem = kKeysSmemFloats * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(bwd_keys_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    bwd_keys_kernel<T><<<dim3((s.N + kTokTile - 1) / kTokTile, BH), kBT, smem, st>>>(
        static_cast<const T*>(a.k), static_cast<const T*>(a.v), s.N, s.d, a.phi, a.dHtot, a.dZtot, a.dphik, a.dk,
        a.dv);
  }
  return cudaGetLastError();
}

// Rows per split of the dW_proj reduction: about two CTAs per SM, whole
// 32-row tiles.
long long wproj_rows_per_split(long long rows) {
  long long per = (rows + 2 * kNumSMs - 1) / (2 * kNumSMs);
  per = (per + kTokTile - 1) / kTokTile * kTokTile;
  return per < kTokTile ? kTokTile : per;
}

template <typename T>
cudaError_t run_wproj(const sla_shape& s, const BwdLayout& L, const float* ol, const void* dout, char* ws,
                      float* dwproj, cudaStream_t st) {
  const long long rows = static_cast<long long>(s.B) * s.H * s.N;
  const long long per = wproj_rows_per_split(rows);
  const int nsplit = static_cast<int>((rows + per - 1) / per);
  float* wpart = reinterpret_cast<float*>(ws + L.wpart);
  bwd_wproj_kernel<T><<<nsplit, kBT, 2 * kTokTile * kLd * sizeof(float), st>>>(ol, static_cast<const T*>(dout), rows,
                                                                               s.d, per, wpart);
  bwd_wproj_sum_kernel<<<(s.d * s.d + kBT - 1) / kBT, kBT, 0, st>>>(wpart, nsplit, s.d, dwproj);
  return cudaGetLastError();
}

}  // namespace

BwdLayout bwd_layout(const sla_shape& s, bool sla_mode) {
  BwdLayout L;
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.status = take(256);
  L.htot = take(BH * kDPad * kDPad * 4);
  L.ztot = take(BH * kDPad * 4);
  L.dhtot = take(BH * kDPad * kDPad * 4);
  L.dztot = take(BH * kDPad * 4);
  L.dphik = take(BH * static_cast<size_t>(s.N) * kDPad * 4);
  if (sla_mode) {
    const size_t rows = BH * static_cast<size_t>(ceil_div(s.N, s.bq));
    const size_t nkv = static_cast<size_t>(ceil_div(s.N, s.bkv));
    const long long flat = static_cast<long long>(BH) * s.N;
    const long long per = wproj_rows_per_split(flat);
    const size_t nsplit = static_cast<size_t>((flat + per - 1) / per);
    L.lists = take(rows * 2 * nkv * 4);
    L.counts = take(rows * 2 * 4);
    L.ol = take(BH * static_cast<size_t>(s.N) * kDPad * 4);
    L.wpart = take(nsplit * kDPad * kDPad * 4);
  }
  L.total = off;
  return L;
}

namespace {

cudaError_t launch_backward_common(const sla_shape& s, const void* q, const void* k, const void* v,
                                   const void* dout, const int32_t* kept, int k_keep, const float* alpha,
                                   const int8_t* labels, const void* wproj, int phi, float* dq, float* dk, float* dv,
                                   float* dalpha, float* dwproj, char* ws, cudaStream_t st) {
  const bool sla_mode = labels != nullptr;
  const BwdLayout L = bwd_layout(s, sla_mode);
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  const size_t nqkv = BH * static_cast<size_t>(s.N) * s.d * sizeof(float);
  const int nq = ceil_div(s.N, s.bq);
  cudaError_t e;
  // accumulators: the key gradients, d alpha and the workspace sums start at zero
  if ((e = cudaMemsetAsync(dk, 0, nqkv, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dv, 0, nqkv, st)) != cudaSuccess) return e;
  if (!sla_mode && (e = cudaMemsetAsync(dalpha, 0, BH * nq * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(ws + L.htot, 0, L.dphik + BH * static_cast<size_t>(s.N) * kDPad * 4 - L.htot, st)) !=
      cudaSuccess)
    return e;
  if (sla_mode) {
    e = launch_labels_to_lists(s, labels, reinterpret_cast<int32_t*>(ws + L.lists),
                               reinterpret_cast<int32_t*>(ws + L.counts), reinterpret_cast<int*>(ws + L.status), st);
    if (e != cudaSuccess) return e;
  }
  BwdArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.dout = dout;
  a.kept = kept;
  a.alpha = alpha;
  a.N = s.N;
  a.d = s.d;
  a.bq = s.bq;
  a.nq = nq;
  a.nkv = ceil_div(s.N, s.bkv);
  a.kk = k_keep;
  a.phi = phi;
  a.scale = 1.0f / sqrtf(static_cast<float>(s.d));
  a.Htot = reinterpret_cast<const float*>(ws + L.htot);
  a.Ztot = reinterpret_cast<const float*>(ws + L.ztot);
  a.dHtot = reinterpret_cast<float*>(ws + L.dhtot);
  a.dZtot = reinterpret_cast<float*>(ws + L.dztot);
  a.dphik = reinterpret_cast<float*>(ws + L.dphik);
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dalpha = dalpha;
  a.status = reinterpret_cast<int*>(ws + L.status);
  a.sla = sla_mode ? 1 : 0;
  a.lists = sla_mode ? reinterpret_cast<const int32_t*>(ws + L.lists) : nullptr;
  a.counts = sla_mode ? reinterpret_cast<const int32_t*>(ws + L.counts) : nullptr;
  a.wproj = static_cast<const __nv_bfloat16*>(wproj);
  a.ol = sla_mode ? reinterpret_cast<float*>(ws + L.ol) : nullptr;
  const bool bf = s.in_dtype == SLA_BF16;
  e = bf ? run_backward<__nv_bfloat16>(s, a, st) : run_backward<float>(s, a, st);
  if (e != cudaSuccess || !sla_mode) return e;
  return bf ? run_wproj<__nv_bfloat16>(s, L, a.ol, dout, ws, dwproj, st)
            : run_wproj<float>(s, L, a.ol, dout, ws, dwproj, st);
}

}  // namespace

cudaError_t launch_backward(const sla_shape& s, const void* q, const void* k, const void* v, const void* dout,
                            const int32_t* kept, int k_keep, const float* alpha, int phi, float* dq, float* dk,
                            float* dv, float* dalpha, char* ws, cudaStream_t st) {
  return launch_backward_common(s, q, k, v, dout, kept, k_keep, alpha, nullptr, nullptr, phi, dq, dk, dv, dalpha,
                                nullptr, ws, st);
}

cudaError_t launch_sla_backward(const sla_shape& s, const void* q, const void* k, const void* v, const void* dout,
                                const int8_t* labels, const void* wproj, int phi, float* dq, float* dk, float* dv,
                                float* dwproj, char* ws, cudaStream_t st) {
  return launch_backward_common(s, q, k, v, dout, nullptr, 0, nullptr, labels, wproj, phi, dq, dk, dv, nullptr,
                                dwproj, ws, st);
}

}  // namespace sla
