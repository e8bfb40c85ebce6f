// backward_tc.cu -- the SLA2 backward on the tensor cores (bf16 inputs,
// d = 128, b_q = 128, b_kv = 64).
//
// Same gradients as backward.cu ("SLA: Beyond Sparsity in Diffusion
// Transformers …" (papernotes.org) 关键设计 4: the sparse part back-propagated
// the FlashAttention way, the linear part through dH_i, dZ_i written as totals
// minus the kept blocks; "SLA2 深度解读 …" (jefxiong.cn) §07: gradients on
// the unquantised inputs), with G_j = dO V_j^T, s = (1 - alpha) / den,
// dden = -(1 - alpha) dO . O_l / den, per query tile i: dH_i = phi(Q_i)^T (s dO_i),
// dZ_i = phi(Q_i)^T dden_i:
//   dS_j = P_j * (alpha G_j - D),  Bx_j = s G_j + dden
//   dQ   = dS K / sqrt(d) + phi'(Q) [ s dO H_tot^T + dden Z_tot^T - sum_j Bx_j phi(K_j) ]
//   dH_tot = sum_i dH_i,  dZ_tot = sum_i dZ_i
// and per key block j, with M_j = dH_tot - sum of dH_i over the tiles i keeping j
// (the kept blocks' linear share regrouped through the tiles' partials):
//   dV_j = sum_i (alpha P_ij)^T dO_i + phi(K_j) M_j
//   dphi(K_j) = V_j M_j^T + dZ_tot - sum_i dZ_i
//   dK_j = sum_i dS_ij^T Q_i / sqrt(d) + phi'(K_j) dphi(K_j)
//
// The per-row quantities (the log2-sum-exp of the kept scores, D, s, dden and
// the row's share of dalpha) come from the attention kernel itself, run once
// more with the upstream gradient (SparseArgs::bwd_rows): it already forms
// O_s, O_l, the row sums and the denominators.  Then:
//   qphi_kernel      phi(Q) as fp16 [BH, N, 128] (the forward's rounding)
//   inv_lists_kernel per key block the query blocks that keep it, ascending
//   bwd_dq_kernel    per query tile: S, G (tcgen05, bf16) per kept block;
//                    dS (bf16), -Bx sigma (fp16) to smem; dQ_s += dS K,
//                    dQ_l += (-Bx sigma) phi(K); then s sigma dO H_tot^T / sigma
//                    and sigma dH_i = phi(Q)^T (s sigma dO), written as -sigma dH_i
//                    in fp16 with dZ_i; epilogue dQ.
//   dh_reduce_kernel dH_tot, dZ_tot: the tiles' partials summed in tile order
//   dh_pack_kernel   tau dH_tot in fp16 (tau a power of two)
//   dalpha_kernel    dalpha per query block: its rows' shares in row order
//   bwd_dkv_kernel   per key block j, with M_j = dH_tot - sum of the dH_i of the
//                    query tiles keeping j (exact regrouping of the kept linear
//                    shares):  dV_j = sum_i (alpha P_ij)^T dO_i + phi(K_j) M_j,
//                    dphi(K_j) = V_j M_j^T + dZ_tot - sum_i dZ_i,
//                    dK_j = sum_i dS_ij^T Q_i / sqrt(d) + phi'(K_j) dphi(K_j):
//                    phase 1 over the tiles keeping j (S, G, then dV^T, dK^T in
//                    TMEM), phase 2 the partials and the totals through
//                    (.) V_j^T and (.)^T phi(K_j)^T, one combined epilogue.
// sigma is the forward's per-head power of two (>= max_e Z_tot[e]); it scales
// Bx, s dO and dH_i into the fp16 range and is divided out exactly.
// Every result is written once in a fixed order: the gradients are the same
// on every run.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "sla_device.cuh"
#include "sla_internal.h"
#include "sla_kernels.h"

namespace sla {

namespace {

// Warps 0..15 work on the 128 rows (or channels) of a tile: warp w takes the
// 32 rows of its TMEM lane quarter w % 4 and column group w / 4 (16 keys of a
// key block, 32 channels in the epilogues), so four warps share each SM
// sub-partition and hide each other's latencies.  Warp 16 issues the TMA
// copies, warp 17 the tensor-core products.
constexpr int kCompute = 512;
constexpr int kTcThreads = kCompute + 64;
constexpr int kProdWarp = 16, kMmaWarp = 17;
constexpr int kRowsT = 128;      // query rows per tile

struct TcArgs {
  int BH, N, nq, nkv, kk, phi;
  float sl2, scale;
  const int32_t* kept;   // [BH, nq, kk]
  const float* alpha;    // [BH, nq]
  const float* rows;     // [BH * N, 8] from the attention kernel's statistics epilogue
  const float* sigma;    // [BH]
  const float* ztot;     // [BH, 128]
  const int32_t* inv;    // [BH, nkv, nq] query blocks keeping each key block
  const int32_t* inv_n;  // [BH, nkv]
  float *dq, *dk, *dv;          // [BH, N, 128]
  __half* dhpart;               // [BH * nq, 128, 128]: -sigma dH_i per query tile
  float* dzpart;                // [BH * nq, 128]: dZ_i per query tile
  const float* dztot;           // [BH, 128]
  const float* tau;             // [BH]: the power of two scaling dH_tot into fp16
  int* status;
  unsigned long long wait_ns;
};

__device__ __forceinline__ int clamp_block(int j, int nkv, int* status, bool report) {
  if (j < 0 || j >= nkv) {
    if (report) report_error(status, SLA_ERR_DEVICE_INDEX);
    return 0;
  }
  return j;
}

__device__ __forceinline__ bool warp_wait_tc(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                             uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status, limit_ns);
  return __all_sync(0xffffffffu, ok) != 0;
}

// Eight 16-bit values of row r into unit u of a 128-byte-swizzled tile.
__device__ __forceinline__ void put_unit(uint8_t* tile, int r, int u, uint32_t a, uint32_t b, uint32_t c,
                                         uint32_t d) {
  *reinterpret_cast<uint4*>(tile + sw128_off(r, u)) = make_uint4(a, b, c, d);
}

// ---------------------------------------------------------------- phi(Q)
// fp16 phi(Q) [rows][128] with the attention kernel's rounding (ELU+1 or the
// channel softmax through ex2.approx).  16 threads per row, 8 channels each.
__global__ void __launch_bounds__(256) qphi_kernel(const __nv_bfloat16* __restrict__ q, __half* __restrict__ out,
                                                   long long rows, int phi) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = idx >> 4;
  const int u = static_cast<int>(idx & 15);
  const bool live = row < rows;
  float x[8];
  {
    uint4 w = make_uint4(0, 0, 0, 0);
    if (live) w = *reinterpret_cast<const uint4*>(q + row * kDPad + 8 * u);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf162(ww[e]);
      x[2 * e] = f.x;
      x[2 * e + 1] = f.y;
    }
  }
  float y[8];
  if (phi == SLA_PHI_SOFTMAX) {
    float mx = x[0];
#pragma unroll
    for (int e = 1; e < 8; ++e) mx = fmaxf(mx, x[e]);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      y[e] = ex2_approx((x[e] - mx) * 1.4426950408889634f);
      sum += y[e];
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = 1.0f / sum;
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] *= inv;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = elu1(x[e]);
  }
  if (live)
    *reinterpret_cast<uint4*>(out + row * kDPad + 8 * u) =
        make_uint4(pack_half2(y[0], y[1]), pack_half2(y[2], y[3]), pack_half2(y[4], y[5]), pack_half2(y[6], y[7]));
}

// ---------------------------------------------------------------- inverse lists
// One warp per (bh, key block j): the query blocks whose kept list holds j,
// ascending (the kept lists are scanned 32 query blocks at a time).
__global__ void __launch_bounds__(256) inv_lists_kernel(const int32_t* __restrict__ kept, int nq, int nkv, int kk,
                                                        int32_t* __restrict__ inv, int32_t* __restrict__ inv_n) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * 8 + warp;
  const long long bh = blockIdx.y;
  if (j >= nkv) return;
  int32_t* dst = inv + (bh * nkv + j) * nq;
  int n = 0;
  for (int i0 = 0; i0 < nq; i0 += 32) {
    const int i = i0 + lane;
    bool hit = false;
    if (i < nq) {
      const int32_t* lst = kept + (bh * nq + i) * kk;
      for (int t = 0; t < kk; ++t) hit = hit || (lst[t] == j);
    }
    const uint32_t m = __ballot_sync(0xffffffffu, hit);
    if (hit) dst[n + __popc(m & ((1u << lane) - 1u))] = i;
    n += __popc(m);
  }
  if (lane == 0) inv_n[bh * nkv + j] = n;
}

// ---------------------------------------------------------------- dQ (query-major)
namespace dq {
constexpr uint32_t OFF_Q = 0;          // bf16 [128 rows] x 2 chunks
constexpr uint32_t OFF_DO = 32768;     // bf16 [128 rows] x 2 chunks
constexpr uint32_t OFF_ST = 65536;     // 2 stages: K | V | phi(K), each 2 chunks of [64 rows][128 B]
constexpr uint32_t STAGE = 49152;
constexpr uint32_t OFF_OPS = OFF_ST + 2 * STAGE;  // dS bf16 [128][64] | -Bx sigma fp16 [128][64]; end: s sigma dO fp16 [128][128]
constexpr uint32_t OFF_BAR = OFF_OPS + 32768;
constexpr uint32_t OFF_MISC = OFF_BAR + 256;
constexpr uint32_t OFF_DD = OFF_MISC + 64;  // dden per row [128] floats
constexpr uint32_t OFF_RED = OFF_DD + 512;  // softmax feature map: [3][4 groups][128 rows] floats
constexpr uint32_t SMEM = OFF_RED + 6144;
static_assert(SMEM <= 232448, "shared memory budget");
// TMEM columns: S_b at 128 b, G_b at 128 b + 64 (b = 0, 1); dQ_s 256; dQ_l 384.
// End phase: s dO H_tot^T at 0, sigma dH_i at 128.
constexpr uint32_t T_DQS = 256, T_DQL = 384, T_HT = 0, T_DH = 128;
enum { B_QD = 0, B_STF = 1, B_STE = 3, B_SGF = 5, B_SGE = 7, B_OPF = 9, B_OPE = 10, B_LOOP = 11, B_ENDL = 12,
       B_SDO = 13, B_END = 14, B_DRAIN = 15, NBAR = 16 };
}  // namespace dq

__global__ void __launch_bounds__(kTcThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmPK, const __grid_constant__ CUtensorMap tmH,
                  const __grid_constant__ CUtensorMap tmPQ, const TcArgs a) {
  using namespace dq;
  extern __shared__ __align__(1024) uint8_t sm[];
  if ((smem_u32(sm) & 1023u) != 0) {
    if (threadIdx.x == 0) report_error(a.status, SLA_ERR_UNSUPPORTED);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  float* ddsh = reinterpret_cast<float*>(sm + OFF_DD);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qb = blockIdx.x % a.nq;
  const int bh = blockIdx.x / a.nq;
  const long long tile = blockIdx.x;
  const int kk = a.kk;
  const int32_t* lst = a.kept + tile * kk;

  if (tid == 0) {
    mbar_init(&bars[B_QD], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[B_STF + s], 1);
      mbar_init(&bars[B_STE + s], 1);
      mbar_init(&bars[B_SGF + s], 1);
      mbar_init(&bars[B_SGE + s], kCompute);
    }
    mbar_init(&bars[B_OPF], kCompute);
    mbar_init(&bars[B_OPE], 1);
    mbar_init(&bars[B_LOOP], 1);
    mbar_init(&bars[B_ENDL], 1);
    mbar_init(&bars[B_SDO], kCompute);
    mbar_init(&bars[B_END], 1);
    mbar_init(&bars[B_DRAIN], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const float sigma = a.sigma[bh];

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      int issued = 0;  // stage loads issued
      mbar_arrive_expect_tx(&bars[B_QD], 65536);
      tma_load_3d(sm + OFF_Q, &tmQ, &bars[B_QD], 0, qb * kRowsT, bh);
      tma_load_3d(sm + OFF_Q + 16384, &tmQ, &bars[B_QD], 64, qb * kRowsT, bh);
      tma_load_3d(sm + OFF_DO, &tmDO, &bars[B_QD], 0, qb * kRowsT, bh);
      tma_load_3d(sm + OFF_DO + 16384, &tmDO, &bars[B_QD], 64, qb * kRowsT, bh);
      for (int n = 0; n < kk; ++n) {
        const int s = n & 1;
        if (n >= 2 && !mbar_wait(&bars[B_STE + s], ((n >> 1) - 1) & 1, abort_flag, a.status, a.wait_ns)) {
          ok = false;
          break;
        }
        const int krow = clamp_block(lst[n], a.nkv, a.status, true) * kBlockKV;
        uint8_t* st = sm + OFF_ST + s * STAGE;
        uint64_t* fb = &bars[B_STF + s];
        mbar_arrive_expect_tx(fb, STAGE);
        tma_load_3d(st, &tmK, fb, 0, krow, bh);
        tma_load_3d(st + 8192, &tmK, fb, 64, krow, bh);
        tma_load_3d(st + 16384, &tmV, fb, 0, krow, bh);
        tma_load_3d(st + 16384 + 8192, &tmV, fb, 64, krow, bh);
        tma_load_3d(st + 32768, &tmPK, fb, 0, krow, bh);
        tma_load_3d(st + 32768 + 8192, &tmPK, fb, 64, krow, bh);
        ++issued;
      }
      bool end_issued = false;
      if (ok && mbar_wait(&bars[B_LOOP], 0, abort_flag, a.status, a.wait_ns)) {
        // every product of the loop is done: the stage area takes H_tot / sigma and phi(Q)
        mbar_arrive_expect_tx(&bars[B_ENDL], 65536);
        tma_load_3d(sm + OFF_ST, &tmH, &bars[B_ENDL], 0, 0, bh);
        tma_load_3d(sm + OFF_ST + 16384, &tmH, &bars[B_ENDL], 64, 0, bh);
        tma_load_3d(sm + OFF_ST + 32768, &tmPQ, &bars[B_ENDL], 0, qb * kRowsT, bh);
        tma_load_3d(sm + OFF_ST + 49152, &tmPQ, &bars[B_ENDL], 64, qb * kRowsT, bh);
        end_issued = true;
      }
      // every issued copy lands before the CTA exits
      mbar_wait_drain(&bars[B_QD], 0);
      for (int g = issued > 2 ? issued - 2 : 0; g < issued; ++g) mbar_wait_drain(&bars[B_STF + (g & 1)], (g >> 1) & 1);
      if (end_issued) mbar_wait_drain(&bars[B_ENDL], 0);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_f16(1, 0, 0, 128, 64);    // Q x K_j^T, dO x V_j^T (bf16, K-major)
      const uint32_t id_qk = idesc_f16(1, 0, 1, 128, 128);  // dS (K-major) x K_j (MN-major), bf16
      const uint32_t id_ql = idesc_f16(0, 0, 1, 128, 128);  // -Bx sigma x phi(K_j) (MN-major), f16
      const uint32_t id_ht = idesc_f16(0, 0, 0, 128, 128);  // s sigma dO (K-major) x H_tot / sigma (K-major), f16
      const uint32_t id_dh = idesc_f16(0, 1, 1, 128, 128);  // phi(Q)^T (MN-major) x s sigma dO (MN-major), f16
      const uint64_t dQd = sdesc_sw128(smem_u32(sm + OFF_Q), 16, 1024);
      const uint64_t dOd = sdesc_sw128(smem_u32(sm + OFF_DO), 16, 1024);
      const uint64_t dStK = sdesc_sw128(smem_u32(sm + OFF_ST), 16, 1024);         // K-major key tiles
      const uint64_t dStMN = sdesc_sw128(smem_u32(sm + OFF_ST), 8192, 1024);      // the same as MN-major
      const uint64_t dOps = sdesc_sw128(smem_u32(sm + OFF_OPS), 16, 1024);        // dS, Bx (K-major, one chunk)
      const uint64_t dSdoK = sdesc_sw128(smem_u32(sm + OFF_OPS), 16, 1024);       // s sigma dO as K-major A
      const uint64_t dSdoMN = sdesc_sw128(smem_u32(sm + OFF_OPS), 16384, 1024);   // ... as MN-major B
      const uint64_t dH = sdesc_sw128(smem_u32(sm + OFF_ST), 16, 1024);           // H_tot / sigma (K-major B)
      const uint64_t dPQ = sdesc_sw128(smem_u32(sm + OFF_ST + 32768), 16384, 1024);  // phi(Q)^T (MN-major A)
      bool ok = mbar_wait(&bars[B_QD], 0, abort_flag, a.status, a.wait_ns);
      auto ops = [&](int m) -> bool {
        if (!mbar_wait(&bars[B_OPF], m & 1, abort_flag, a.status, a.wait_ns)) return false;
        tc_fence_after();
        const uint32_t so = ((m & 1) * STAGE) >> 4;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)  // K = 64 keys: A +32 B, B +2048 B per 16
          mma_f16_ss(tmem + T_DQS, dOps + k4 * 2u, dStMN + so + k4 * 128u, id_qk, (m > 0 || k4 > 0) ? 1u : 0u);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)
          mma_f16_ss(tmem + T_DQL, dOps + (16384u >> 4) + k4 * 2u, dStMN + so + (32768u >> 4) + k4 * 128u, id_ql,
                     (m > 0 || k4 > 0) ? 1u : 0u);
        mma_commit(&bars[B_OPE]);
        mma_commit(&bars[B_STE + (m & 1)]);
        return true;
      };
      for (int n = 0; ok && n < kk; ++n) {
        const int b = n & 1;
        if (!mbar_wait(&bars[B_STF + b], (n >> 1) & 1, abort_flag, a.status, a.wait_ns)) {
          ok = false;
          break;
        }
        if (n >= 2 && !mbar_wait(&bars[B_SGE + b], ((n >> 1) - 1) & 1, abort_flag, a.status, a.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t so = (b * STAGE) >> 4;
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) {
          const uint32_t oa = ((k8 >> 2) * 16384u + (k8 & 3) * 32u) >> 4;
          const uint32_t ob = ((k8 >> 2) * 8192u + (k8 & 3) * 32u) >> 4;
          mma_f16_ss(tmem + 128 * b, dQd + oa, dStK + so + ob, id_s, k8 > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) {
          const uint32_t oa = ((k8 >> 2) * 16384u + (k8 & 3) * 32u) >> 4;
          const uint32_t ob = (16384u + (k8 >> 2) * 8192u + (k8 & 3) * 32u) >> 4;
          mma_f16_ss(tmem + 128 * b + 64, dOd + oa, dStK + so + ob, id_s, k8 > 0 ? 1u : 0u);
        }
        mma_commit(&bars[B_SGF + b]);
        if (n >= 1 && !ops(n - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && kk > 0) ok = ops(kk - 1);
      if (ok) mma_commit(&bars[B_LOOP]);
      if (ok && mbar_wait(&bars[B_ENDL], 0, abort_flag, a.status, a.wait_ns) &&
          mbar_wait(&bars[B_SDO], 0, abort_flag, a.status, a.wait_ns)) {
        tc_fence_after();
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) {  // s dO H_tot^T: K = 128 channels
          const uint32_t o = ((k8 >> 2) * 16384u + (k8 & 3) * 32u) >> 4;
          mma_f16_ss(tmem + T_HT, dSdoK + o, dH + o, id_ht, k8 > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8)  // sigma dH_i: K = 128 rows, +2048 B per 16
          mma_f16_ss(tmem + T_DH, dPQ + k8 * 128u, dSdoMN + k8 * 128u, id_dh, k8 > 0 ? 1u : 0u);
        mma_commit(&bars[B_END]);
      }
      mma_commit(&bars[B_DRAIN]);
      mbar_wait_drain(&bars[B_DRAIN], 0);
    }
  } else {
    // ------------------------------------------------------------ rows (warps 0..15)
    const int q4 = warp & 3, g = warp >> 2;
    const int r = q4 * 32 + lane;  // tile row = TMEM lane
    const uint32_t lrow = static_cast<uint32_t>(q4 * 32) << 16;
    const int tok = qb * kRowsT + r;
    const bool valid = tok < a.N;
    float lse2 = 0.0f, D = 0.0f, sr = 0.0f, dd = 0.0f;
    if (valid) {
      const float4 st = *reinterpret_cast<const float4*>(a.rows + (static_cast<long long>(bh) * a.N + tok) * 8);
      lse2 = st.x;
      D = st.y;
      sr = st.z;
      dd = st.w;
    }
    const float alpha = a.alpha[tile];
    const bool tail = (a.N & (kBlockKV - 1)) != 0;
    bool ok = true;
    uint8_t* opS = sm + OFF_OPS;
    uint8_t* opB = sm + OFF_OPS + 16384;
    for (int n = 0; n < kk; ++n) {
      const int b = n & 1;
      ok = ok && warp_wait_tc(&bars[B_SGF + b], (n >> 1) & 1, abort_flag, a.status, a.wait_ns);
      if (!ok) break;
      tc_fence_after();
      const int j = clamp_block(lst[n], a.nkv, a.status, false);
      const int nvalid = (tail && j == a.nkv - 1) ? a.N - j * kBlockKV : kBlockKV;
      float sv[16], gv[16];
      tmem_ld16(tmem + lrow + 128 * b + 16 * g, sv);
      tmem_ld16(tmem + lrow + 128 * b + 64 + 16 * g, gv);
      tmem_wait_ld();
      uint32_t pS[8], pB[8];
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        float ds[2], bx[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool kv = valid && (16 * g + c + e < nvalid);
          const float p = kv ? ex2_approx(fmaf(sv[c + e], a.sl2, -lse2)) : 0.0f;
          ds[e] = p * fmaf(alpha, gv[c + e], -D);
          bx[e] = kv ? -fmaf(sr, gv[c + e], dd) * sigma : 0.0f;
        }
        pS[c / 2] = pack_bf162(ds[0], ds[1]);
        pB[c / 2] = pack_half2(bx[0], bx[1]);
      }
      tc_fence_before();
      mbar_arrive(&bars[B_SGE + b]);
      ok = ok && (n == 0 || warp_wait_tc(&bars[B_OPE], (n - 1) & 1, abort_flag, a.status, a.wait_ns));
      if (!ok) break;
      put_unit(opS, r, 2 * g, pS[0], pS[1], pS[2], pS[3]);
      put_unit(opS, r, 2 * g + 1, pS[4], pS[5], pS[6], pS[7]);
      put_unit(opB, r, 2 * g, pB[0], pB[1], pB[2], pB[3]);
      put_unit(opB, r, 2 * g + 1, pB[4], pB[5], pB[6], pB[7]);
      fence_proxy_async_smem();
      mbar_arrive(&bars[B_OPF]);
    }
    // s sigma dO (fp16, channels 32 g ..) over the operand tiles once the loop's products
    // are done (the Q and dO tiles read from here on landed on B_QD, long complete)
    ok = ok && warp_wait_tc(&bars[B_LOOP], 0, abort_flag, a.status, a.wait_ns);
    ok = ok && warp_wait_tc(&bars[B_QD], 0, abort_flag, a.status, a.wait_ns);
    if (ok) {
      const float f = sr * sigma;
#pragma unroll
      for (int u4 = 0; u4 < 4; ++u4) {
        const int u = (g & 1) * 4 + u4;
        const uint32_t ch = static_cast<uint32_t>(g >> 1) * 16384u;
        const uint4 w = *reinterpret_cast<const uint4*>(sm + OFF_DO + ch + sw128_off(r, u));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        uint32_t o4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 gg = unpack_bf162(ww[e]);
          o4[e] = pack_half2(gg.x * f, gg.y * f);
        }
        put_unit(sm + OFF_OPS + ch, r, u, o4[0], o4[1], o4[2], o4[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars[B_SDO]);
    }
    if (g == 0) ddsh[r] = dd;
    named_bar_sync(1, kCompute);
    // dZ_i[e] = sum over the rows of phi(Q)[row][e] dden[row], e = r (phi(Q) tile in smem)
    ok = ok && warp_wait_tc(&bars[B_ENDL], 0, abort_flag, a.status, a.wait_ns);
    if (ok && g == 0) {
      const int e = r, ch = e >> 6, u = (e & 63) >> 3, w = e & 7;
      float z = 0.0f;
      for (int rr = 0; rr < kRowsT; ++rr) {
        const __half* hp =
            reinterpret_cast<const __half*>(sm + OFF_ST + 32768 + ch * 16384u + sw128_off(rr, u)) + w;
        z = fmaf(__half2float(*hp), ddsh[rr], z);
      }
      a.dzpart[tile * kDPad + e] = z;
    }
    ok = ok && warp_wait_tc(&bars[B_END], 0, abort_flag, a.status, a.wait_ns);
    if (ok) tc_fence_after();
    const float inv_sigma = 1.0f / sigma;  // exact: a power of two
    if (ok) {
      // -sigma dH_i as fp16 (the key kernel subtracts the tiles keeping each key
      // block from the totals): lane e = r, columns c = 32 g ..
      __half* dh = a.dhpart + (tile * kDPad + r) * kDPad + 32 * g;
      float hv[32];
      tmem_ld32(tmem + lrow + T_DH + 32 * g, hv);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; c += 8)
        *reinterpret_cast<uint4*>(dh + c) = make_uint4(pack_half2(-hv[c], -hv[c + 1]), pack_half2(-hv[c + 2], -hv[c + 3]),
                                                       pack_half2(-hv[c + 4], -hv[c + 5]),
                                                       pack_half2(-hv[c + 6], -hv[c + 7]));
    }
    // dQ of row r, channels 32 g + 16 h ..: scale dQ_s + phi'(Q) (dQ_l / sigma + s dO H_tot^T + dden Z_tot)
    const float* zt = a.ztot + static_cast<long long>(bh) * kDPad;
    const bool have = kk > 0;
    auto q16 = [&](int h, float* x) {  // 16 channels of Q row r from the smem tile
#pragma unroll
      for (int u2 = 0; u2 < 2; ++u2) {
        const uint4 w = *reinterpret_cast<const uint4*>(sm + OFF_Q + (g >> 1) * 16384u +
                                                        sw128_off(r, (g & 1) * 4 + 2 * h + u2));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack_bf162(ww[e]);
          x[8 * u2 + 2 * e] = f.x;
          x[8 * u2 + 2 * e + 1] = f.y;
        }
      }
    };
    auto gphi16 = [&](int h, float* gp) {  // the gradient reaching phi(Q), 16 channels
      float l[16], hh[16];
      tmem_ld16(tmem + lrow + T_DQL + 32 * g + 16 * h, l);
      tmem_ld16(tmem + lrow + T_HT + 32 * g + 16 * h, hh);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 16; ++c) gp[c] = (have ? l[c] * inv_sigma : 0.0f) + hh[c] + dd * zt[32 * g + 16 * h + c];
    };
    // the softmax feature map: phi'(q) gp = phi (gp - sum_c phi_c gp_c); the row's
    // max, sum and dot are combined over the four column groups in smem
    const bool smx = a.phi == SLA_PHI_SOFTMAX;
    float mx = -INFINITY, inv_sum = 0.0f, dot = 0.0f;
    if (smx) {
      float* red = reinterpret_cast<float*>(sm + OFF_RED);
      float x[16];
      float pm = -INFINITY;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        q16(h, x);
#pragma unroll
        for (int c = 0; c < 16; ++c) pm = fmaxf(pm, x[c]);
      }
      red[g * 128 + r] = pm;
      named_bar_sync(1, kCompute);
      mx = fmaxf(fmaxf(red[r], red[128 + r]), fmaxf(red[256 + r], red[384 + r]));
      float ps = 0.0f;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        q16(h, x);
#pragma unroll
        for (int c = 0; c < 16; ++c) ps += expf(x[c] - mx);
      }
      red[512 + g * 128 + r] = ps;
      named_bar_sync(1, kCompute);
      inv_sum = 1.0f / ((red[512 + r] + red[640 + r]) + (red[768 + r] + red[896 + r]));
      float pd = 0.0f;
      if (ok) {
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          float gp[16];
          q16(h, x);
          gphi16(h, gp);
#pragma unroll
          for (int c = 0; c < 16; ++c) pd = fmaf(expf(x[c] - mx) * inv_sum, gp[c], pd);
        }
      }
      red[1024 + g * 128 + r] = pd;
      named_bar_sync(1, kCompute);
      dot = (red[1024 + r] + red[1152 + r]) + (red[1280 + r] + red[1408 + r]);
    }
    if (ok) {
      float* dqr = a.dq + (static_cast<long long>(bh) * a.N + tok) * kDPad + 32 * g;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float gp[16], sq[16], x[16];
        q16(h, x);
        gphi16(h, gp);
        tmem_ld16(tmem + lrow + T_DQS + 32 * g + 16 * h, sq);
        tmem_wait_ld();
        float o[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float dphi = smx ? expf(x[c] - mx) * inv_sum * (gp[c] - dot) : gp[c] * (x[c] > 0.0f ? 1.0f : expf(x[c]));
          o[c] = (have ? sq[c] * a.scale : 0.0f) + dphi;
        }
        if (valid) {
#pragma unroll
          for (int c = 0; c < 16; c += 4)
            *reinterpret_cast<float4*>(dqr + 16 * h + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dK, dV (key-major)
// One CTA per key block j of a head (64 keys).  With M_j = dH_tot minus the
// dH_i of the query tiles i keeping j:
//   dV_j = sum_i (alpha_i P_ij)^T dO_i + phi(K_j) M_j
//   dphi(K_j) = V_j M_j^T + dZ_tot - sum_i dZ_i,  dK_j = sum_i dS_ij^T Q_i / sqrt(d) + phi'(K_j) dphi(K_j)
// (the linear shares through the query tiles' partials, so the loop over the
// tiles keeping j needs S, G, P and dS only).  Phase 1, per such tile i (two
// operand stages, two S/G buffers): S = Q_i K_j^T, G = dO_i V_j^T; the row warps
// write dS and alpha P (bf16); dV^T += dO_i^T (alpha P), dK^T += Q_i^T dS.  Phase 2:
// the tiles' -sigma dH_i (fp16, from bwd_dq_kernel) and tau dH_tot through
// (.) V16_j^T and (.)^T phi(K_j)^T, four 32 KB slots in the stage area.  The
// epilogue combines everything; each gradient is written once.
namespace dkv {
constexpr uint32_t OFF_K = 0;          // K_j bf16 | V_j bf16 | V_j fp16 | phi(K_j) fp16: each 2 chunks of [64 rows][128 B]
constexpr uint32_t OFF_V = 16384;
constexpr uint32_t OFF_V16 = 32768;
constexpr uint32_t OFF_PK = 49152;
constexpr uint32_t OFF_ST = 65536;     // phase 1: 2 stages of Q_i | dO_i (2 chunks of [128 rows][128 B] each)
constexpr uint32_t STAGE = 65536;      // phase 2: 4 slots of one [128][128] fp16 tile
constexpr uint32_t SLOT = 32768;
constexpr uint32_t OFF_OPS = OFF_ST + 2 * STAGE;  // dS bf16 | alpha P bf16, each [128 rows][64 keys]; epilogue reductions
constexpr uint32_t OFF_BAR = OFF_OPS + 32768;
constexpr uint32_t OFF_MISC = OFF_BAR + 256;
constexpr uint32_t SMEM = OFF_MISC + 64;
static_assert(SMEM <= 232448, "shared memory budget");
// TMEM: phase 1 S_b at 128 b, G_b at 128 b + 64; then tau dH_tot V^T at 0, (tau dH_tot)^T phi(K)^T at 64;
// dV^T 256, dK^T 320, the tiles' -sigma dH_i V^T 384, (-sigma dH_i)^T phi(K)^T 448
constexpr uint32_t T_TP = 0, T_TV = 64, T_DV = 256, T_DK = 320, T_KP = 384, T_KV = 448;
enum { B_KV = 0, B_STF = 1, B_STE = 3, B_SGF = 5, B_SGE = 7, B_OPF = 9, B_OPE = 10, B_SLOOP = 11, B_LF = 12,
       B_LE = 16, B_DONE = 20, B_DRAIN = 21, NBAR = 22 };
static_assert(NBAR * 8 <= 256, "barrier area");
}  // namespace dkv

__global__ void __launch_bounds__(kTcThreads, 1)
    bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmV16, const __grid_constant__ CUtensorMap tmPK,
                   const __grid_constant__ CUtensorMap tmDHi, const __grid_constant__ CUtensorMap tmDH,
                   const TcArgs a) {
  using namespace dkv;
  extern __shared__ __align__(1024) uint8_t sm[];
  if ((smem_u32(sm) & 1023u) != 0) {
    if (threadIdx.x == 0) report_error(a.status, SLA_ERR_UNSUPPORTED);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x % a.nkv;
  const int bh = blockIdx.x / a.nkv;
  const long long kb = static_cast<long long>(bh) * a.nkv + j;
  int cnt = a.inv_n[kb];
  if (cnt < 0 || cnt > a.nq) cnt = 0;
  const int32_t* il = a.inv + kb * a.nq;
  auto tile_of = [&](int n) -> int {
    const int i = il[n];
    return (i < 0 || i >= a.nq) ? 0 : i;
  };

  if (tid == 0) {
    for (int b = 0; b < NBAR; ++b)
      mbar_init(&bars[b], (b == B_OPF || b == B_SGE || b == B_SGE + 1) ? kCompute : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const float sigma = a.sigma[bh];

  if (warp == kProdWarp) {
    if (lane == 0) {
      bool ok = true;
      int issued = 0, lissued = 0;
      mbar_arrive_expect_tx(&bars[B_KV], 65536);
      const int krow = j * kBlockKV;
      tma_load_3d(sm + OFF_K, &tmK, &bars[B_KV], 0, krow, bh);
      tma_load_3d(sm + OFF_K + 8192, &tmK, &bars[B_KV], 64, krow, bh);
      tma_load_3d(sm + OFF_V, &tmV, &bars[B_KV], 0, krow, bh);
      tma_load_3d(sm + OFF_V + 8192, &tmV, &bars[B_KV], 64, krow, bh);
      tma_load_3d(sm + OFF_V16, &tmV16, &bars[B_KV], 0, krow, bh);
      tma_load_3d(sm + OFF_V16 + 8192, &tmV16, &bars[B_KV], 64, krow, bh);
      tma_load_3d(sm + OFF_PK, &tmPK, &bars[B_KV], 0, krow, bh);
      tma_load_3d(sm + OFF_PK + 8192, &tmPK, &bars[B_KV], 64, krow, bh);
      for (int n = 0; n < cnt; ++n) {
        const int s = n & 1;
        if (n >= 2 && !mbar_wait(&bars[B_STE + s], ((n >> 1) - 1) & 1, abort_flag, a.status, a.wait_ns)) {
          ok = false;
          break;
        }
        const int i = tile_of(n);
        uint8_t* st = sm + OFF_ST + s * STAGE;
        uint64_t* fb = &bars[B_STF + s];
        mbar_arrive_expect_tx(fb, STAGE);
        tma_load_3d(st, &tmQ, fb, 0, i * kRowsT, bh);
        tma_load_3d(st + 16384, &tmQ, fb, 64, i * kRowsT, bh);
        tma_load_3d(st + 32768, &tmDO, fb, 0, i * kRowsT, bh);
        tma_load_3d(st + 49152, &tmDO, fb, 64, i * kRowsT, bh);
        ++issued;
      }
      // phase 2 once every phase-1 product is done: the tiles' partials, then the totals
      if (ok && mbar_wait(&bars[B_SLOOP], 0, abort_flag, a.status, a.wait_ns)) {
        for (int m = 0; m <= cnt; ++m) {
          const int sl = m & 3;
          if (m >= 4 && !mbar_wait(&bars[B_LE + sl], ((m >> 2) - 1) & 1, abort_flag, a.status, a.wait_ns)) break;
          uint8_t* dst = sm + OFF_ST + sl * SLOT;
          uint64_t* fb = &bars[B_LF + sl];
          mbar_arrive_expect_tx(fb, SLOT);
          if (m < cnt) {
            const int t = bh * a.nq + tile_of(m);
            tma_load_3d(dst, &tmDHi, fb, 0, 0, t);
            tma_load_3d(dst + 16384, &tmDHi, fb, 64, 0, t);
          } else {
            tma_load_3d(dst, &tmDH, fb, 0, 0, bh);
            tma_load_3d(dst + 16384, &tmDH, fb, 64, 0, bh);
          }
          ++lissued;
        }
      }
      // every issued copy lands before the CTA exits
      mbar_wait_drain(&bars[B_KV], 0);
      for (int g2 = issued > 2 ? issued - 2 : 0; g2 < issued; ++g2)
        mbar_wait_drain(&bars[B_STF + (g2 & 1)], (g2 >> 1) & 1);
      for (int g2 = lissued > 4 ? lissued - 4 : 0; g2 < lissued; ++g2)
        mbar_wait_drain(&bars[B_LF + (g2 & 3)], (g2 >> 2) & 1);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t id_s = idesc_f16(1, 0, 0, 128, 64);   // Q_i K_j^T, dO_i V_j^T (bf16, K-major)
      const uint32_t id_t = idesc_f16(1, 1, 1, 128, 64);   // dO^T (alpha P), Q^T dS (bf16, both MN-major)
      const uint32_t id_lp = idesc_f16(0, 0, 0, 128, 64);  // T V16_j^T (f16, both K-major)
      const uint32_t id_lv = idesc_f16(0, 1, 0, 128, 64);  // T^T (MN-major) phi(K_j)^T (K-major), f16
      const uint64_t dKd = sdesc_sw128(smem_u32(sm + OFF_K), 16, 1024);
      const uint64_t dStK = sdesc_sw128(smem_u32(sm + OFF_ST), 16, 1024);
      const uint64_t dStMN = sdesc_sw128(smem_u32(sm + OFF_ST), 16384, 1024);
      const uint64_t dOpsMN = sdesc_sw128(smem_u32(sm + OFF_OPS), 16, 1024);  // N = 64 fits one atom
      bool ok = mbar_wait(&bars[B_KV], 0, abort_flag, a.status, a.wait_ns);
      auto ops = [&](int m) -> bool {
        if (!mbar_wait(&bars[B_OPF], m & 1, abort_flag, a.status, a.wait_ns)) return false;
        tc_fence_after();
        const uint32_t so = ((m & 1) * STAGE) >> 4;
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) {  // K = 128 rows, +2048 B per 16
          const uint32_t acc = (m > 0 || k8 > 0) ? 1u : 0u;
          mma_f16_ss(tmem + T_DV, dStMN + so + (32768u >> 4) + k8 * 128u, dOpsMN + (16384u >> 4) + k8 * 128u, id_t,
                     acc);
          mma_f16_ss(tmem + T_DK, dStMN + so + k8 * 128u, dOpsMN + k8 * 128u, id_t, acc);
        }
        mma_commit(&bars[B_OPE]);
        mma_commit(&bars[B_STE + (m & 1)]);
        return true;
      };
      for (int n = 0; ok && n < cnt; ++n) {
        const int b = n & 1;
        if (!mbar_wait(&bars[B_STF + b], (n >> 1) & 1, abort_flag, a.status, a.wait_ns)) {
          ok = false;
          break;
        }
        if (n >= 2 && !mbar_wait(&bars[B_SGE + b], ((n >> 1) - 1) & 1, abort_flag, a.status, a.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t so = (b * STAGE) >> 4;
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) {  // M = 128 rows, N = 64 keys, K = 128 channels
          const uint32_t oa = ((k8 >> 2) * 16384u + (k8 & 3) * 32u) >> 4;
          const uint32_t ob = ((k8 >> 2) * 8192u + (k8 & 3) * 32u) >> 4;
          mma_f16_ss(tmem + 128 * b, dStK + so + oa, dKd + ob, id_s, k8 > 0 ? 1u : 0u);
          mma_f16_ss(tmem + 128 * b + 64, dStK + so + (32768u >> 4) + oa, dKd + (16384u >> 4) + ob, id_s,
                     k8 > 0 ? 1u : 0u);
        }
        mma_commit(&bars[B_SGF + b]);
        if (n >= 1 && !ops(n - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && cnt > 0) ok = ops(cnt - 1);
      if (ok) mma_commit(&bars[B_SLOOP]);
      for (int m = 0; ok && m <= cnt; ++m) {
        const int sl = m & 3;
        if (!mbar_wait(&bars[B_LF + sl], (m >> 2) & 1, abort_flag, a.status, a.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t so = (sl * SLOT) >> 4;
        const bool tot = m == cnt;
        const uint32_t cp = tot ? T_TP : T_KP, cv = tot ? T_TV : T_KV;
#pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) {  // M = 128 (e, then c), N = 64 keys, K = 128
          const uint32_t acc = ((!tot && m > 0) || k8 > 0) ? 1u : 0u;
          const uint32_t oa = ((k8 >> 2) * 16384u + (k8 & 3) * 32u) >> 4;
          const uint32_t ob = ((k8 >> 2) * 8192u + (k8 & 3) * 32u) >> 4;
          mma_f16_ss(tmem + cp, dStK + so + oa, dKd + (32768u >> 4) + ob, id_lp, acc);
          mma_f16_ss(tmem + cv, dStMN + so + k8 * 128u, dKd + (49152u >> 4) + ob, id_lv, acc);
        }
        mma_commit(&bars[B_LE + sl]);
      }
      if (ok) mma_commit(&bars[B_DONE]);
      mma_commit(&bars[B_DRAIN]);
      mbar_wait_drain(&bars[B_DRAIN], 0);
    }
  } else {
    // warp w: rows (epilogue: channels) 32 (w % 4) .., keys 16 (w / 4) .. of the block
    const int q4 = warp & 3, g = warp >> 2;
    const int r = q4 * 32 + lane;
    const uint32_t lrow = static_cast<uint32_t>(q4 * 32) << 16;
    const bool tail = (a.N & (kBlockKV - 1)) != 0;
    const int nvalid = (tail && j == a.nkv - 1) ? a.N - j * kBlockKV : kBlockKV;
    bool ok = true;
    uint8_t* opS = sm + OFF_OPS;
    uint8_t* opP = sm + OFF_OPS + 16384;
    for (int n = 0; n < cnt; ++n) {
      const int i = tile_of(n);
      const int tok = i * kRowsT + r;
      const bool valid = tok < a.N;
      float lse2 = 0.0f, D = 0.0f;
      if (valid) {
        const float2 st = *reinterpret_cast<const float2*>(a.rows + (static_cast<long long>(bh) * a.N + tok) * 8);
        lse2 = st.x;
        D = st.y;
      }
      const float alpha = a.alpha[static_cast<long long>(bh) * a.nq + i];
      const int b = n & 1;
      ok = ok && warp_wait_tc(&bars[B_SGF + b], (n >> 1) & 1, abort_flag, a.status, a.wait_ns);
      if (!ok) break;
      tc_fence_after();
      float sv[16], gv[16];
      tmem_ld16(tmem + lrow + 128 * b + 16 * g, sv);
      tmem_ld16(tmem + lrow + 128 * b + 64 + 16 * g, gv);
      tmem_wait_ld();
      uint32_t pS[8], pP[8];
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        float ds[2], ap[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool kv = valid && (16 * g + c + e < nvalid);
          const float p = kv ? ex2_approx(fmaf(sv[c + e], a.sl2, -lse2)) : 0.0f;
          ds[e] = p * fmaf(alpha, gv[c + e], -D);
          ap[e] = alpha * p;
        }
        pS[c / 2] = pack_bf162(ds[0], ds[1]);
        pP[c / 2] = pack_bf162(ap[0], ap[1]);
      }
      tc_fence_before();
      mbar_arrive(&bars[B_SGE + b]);
      ok = ok && (n == 0 || warp_wait_tc(&bars[B_OPE], (n - 1) & 1, abort_flag, a.status, a.wait_ns));
      if (!ok) break;
      put_unit(opS, r, 2 * g, pS[0], pS[1], pS[2], pS[3]);
      put_unit(opS, r, 2 * g + 1, pS[4], pS[5], pS[6], pS[7]);
      put_unit(opP, r, 2 * g, pP[0], pP[1], pP[2], pP[3]);
      put_unit(opP, r, 2 * g + 1, pP[4], pP[5], pP[6], pP[7]);
      fence_proxy_async_smem();
      mbar_arrive(&bars[B_OPF]);
    }
    // epilogue: lane = channel c; keys 16 g .. of the block (the K tile read here
    // landed on B_KV, long complete)
    ok = ok && warp_wait_tc(&bars[B_DONE], 0, abort_flag, a.status, a.wait_ns);
    ok = ok && warp_wait_tc(&bars[B_KV], 0, abort_flag, a.status, a.wait_ns);
    if (ok) tc_fence_after();
    const int c = r;
    const bool have = cnt > 0;
    const float inv_sigma = 1.0f / sigma, inv_tau = 1.0f / a.tau[bh];  // exact: powers of two
    float zc = a.dztot[static_cast<long long>(bh) * kDPad + c];
    for (int n = 0; n < cnt; ++n) zc -= a.dzpart[(static_cast<long long>(bh) * a.nq + tile_of(n)) * kDPad + c];
    // the key values k[key][c] of this thread's 16 keys (bf16 tile in smem), and
    // dphi(k) = (tau dH_tot) V^T / tau + (-sigma sum dH_i) V^T / sigma + dZ_tot - sum dZ_i
    float kx[16], dphi[16];
    {
      float tp[16], kp[16];
      if (ok) {
        tmem_ld16(tmem + lrow + T_TP + 16 * g, tp);
        tmem_ld16(tmem + lrow + T_KP + 16 * g, kp);
        tmem_wait_ld();
      }
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const int key = 16 * g + x;
        const __nv_bfloat16* kp16 = reinterpret_cast<const __nv_bfloat16*>(
            sm + OFF_K + (c >> 6) * 8192u + sw128_off(key, (c & 63) >> 3)) + (c & 7);
        kx[x] = __bfloat162float(*kp16);
        dphi[x] = ok ? tp[x] * inv_tau + (have ? kp[x] * inv_sigma : 0.0f) + zc : 0.0f;
      }
    }
    const bool smx = a.phi == SLA_PHI_SOFTMAX;
    if (smx) {
      // phi'(k) dphi = f (dphi - sum_c f_c dphi_c), f the softmax of the key over its
      // 128 channels (the lanes of the four warps that share g): kx becomes f, dphi
      // becomes phi'(k) dphi
      float* red = reinterpret_cast<float*>(sm + OFF_OPS);  // [3][4 groups][4 quarters][16 keys]
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        float m = kx[x];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) red[(g * 4 + q4) * 16 + x] = m;
      }
      named_bar_sync(1, kCompute);
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const float* rr = red + g * 64 + x;
        float e = expf(kx[x] - fmaxf(fmaxf(rr[0], rr[16]), fmaxf(rr[32], rr[48])));
        kx[x] = e;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
        if (lane == 0) red[256 + (g * 4 + q4) * 16 + x] = e;
      }
      named_bar_sync(1, kCompute);
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const float* rr = red + 256 + g * 64 + x;
        kx[x] /= (rr[0] + rr[16]) + (rr[32] + rr[48]);
        float dd = kx[x] * dphi[x];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dd += __shfl_xor_sync(0xffffffffu, dd, o);
        if (lane == 0) red[512 + (g * 4 + q4) * 16 + x] = dd;
      }
      named_bar_sync(1, kCompute);
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const float* rr = red + 512 + g * 64 + x;
        dphi[x] = kx[x] * (dphi[x] - ((rr[0] + rr[16]) + (rr[32] + rr[48])));
      }
    } else {
#pragma unroll
      for (int x = 0; x < 16; ++x) dphi[x] *= kx[x] > 0.0f ? 1.0f : expf(kx[x]);
    }
    if (ok) {
      const long long base = (static_cast<long long>(bh) * a.N + static_cast<long long>(j) * kBlockKV) * kDPad + c;
      {
        float dkx[16];
        tmem_ld16(tmem + lrow + T_DK + 16 * g, dkx);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int key = 16 * g + x;
          if (key < nvalid) a.dk[base + static_cast<long long>(key) * kDPad] = (have ? dkx[x] * a.scale : 0.0f) + dphi[x];
        }
      }
      float dvx[16], tv[16], kv2[16];
      tmem_ld16(tmem + lrow + T_DV + 16 * g, dvx);
      tmem_ld16(tmem + lrow + T_TV + 16 * g, tv);
      tmem_ld16(tmem + lrow + T_KV + 16 * g, kv2);
      tmem_wait_ld();
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const int key = 16 * g + x;
        if (key < nvalid)
          a.dv[base + static_cast<long long>(key) * kDPad] =
              (have ? dvx[x] : 0.0f) + tv[x] * inv_tau + (have ? kv2[x] * inv_sigma : 0.0f);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- reductions
// grid (64, BH): dH_tot[bh][e][c] and dZ_tot[bh][e] as the tiles' partials summed in
// tile order (the dH partials are -sigma dH_i in fp16).
__global__ void __launch_bounds__(256) dh_reduce_kernel(const __half* __restrict__ dhpart,
                                                        const float* __restrict__ dzpart,
                                                        const float* __restrict__ sigma, int nq,
                                                        float* __restrict__ dhtot, float* __restrict__ dztot) {
  const long long bh = blockIdx.y;
  const int x = blockIdx.x * 256 + threadIdx.x;  // element of the 128 x 128 block
  const __half* src = dhpart + bh * nq * kDPad * kDPad + x;
  float t = 0.0f;
  for (int i = 0; i < nq; ++i) t += __half2float(src[static_cast<long long>(i) * kDPad * kDPad]);
  dhtot[bh * kDPad * kDPad + x] = -t / sigma[bh];  // exact division: sigma is a power of two
  if (blockIdx.x == 0 && threadIdx.x < kDPad) {
    const float* zs = dzpart + bh * nq * kDPad + threadIdx.x;
    float z = 0.0f;
    for (int i = 0; i < nq; ++i) z += zs[static_cast<long long>(i) * kDPad];
    dztot[bh * kDPad + threadIdx.x] = z;
  }
}

// One block per head: tau = a power of two with tau max|dH_tot| < 2^14 (1 if dH_tot = 0)
// and the fp16 copy tau dH_tot for the key kernel's totals products.
__global__ void __launch_bounds__(256) dh_pack_kernel(const float* __restrict__ dhtot, __half* __restrict__ dh16,
                                                      float* __restrict__ tau) {
  __shared__ float red[8];
  const long long bh = blockIdx.x;
  const float* src = dhtot + bh * kDPad * kDPad;
  float m = 0.0f;
  for (int x = threadIdx.x; x < kDPad * kDPad; x += 256) m = fmaxf(m, fabsf(src[x]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = 0.0f;
#pragma unroll
  for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w]);
  int ex = 0;
  if (m > 0.0f) frexpf(m, &ex);  // m < 2^ex
  const float t = m > 0.0f ? ldexpf(1.0f, 14 - ex) : 1.0f;
  if (threadIdx.x == 0) tau[bh] = t;
  for (int x = threadIdx.x; x < kDPad * kDPad; x += 256) dh16[bh * kDPad * kDPad + x] = __float2half_rn(src[x] * t);
}

// One warp per (bh, query block): dalpha = its rows' dO . (O_s - O_l), lane-strided then a fixed tree.
__global__ void __launch_bounds__(256) dalpha_kernel(const float* __restrict__ rows, int N, int nq, long long ntile,
                                                     float* __restrict__ dalpha) {
  const long long t = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= ntile) return;
  const long long bh = t / nq;
  const int i = static_cast<int>(t % nq);
  float s = 0.0f;
  for (int r = lane; r < kRowsT; r += 32) {
    const int tok = i * kRowsT + r;
    if (tok < N) s += rows[(bh * N + tok) * 8 + 4];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) dalpha[t] = s;
}

}  // namespace

BwdTcLayout bwd_tc_layout(const sla_shape& s) {
  BwdTcLayout L;
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  const size_t N = static_cast<size_t>(s.N);
  const size_t nq = static_cast<size_t>(ceil_div(s.N, s.bq)), nkv = static_cast<size_t>(ceil_div(s.N, s.bkv));
  L.fwd = ws_layout(s, SLA_MODE_SLA2_TOPK);
  size_t off = L.fwd.total;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.rows = take(BH * N * 8 * 4);
  L.phiq = take(BH * N * kDPad * 2);
  L.inv = take(BH * nkv * nq * 4);
  L.inv_n = take(BH * nkv * 4);
  L.dhpart = take(BH * nq * kDPad * kDPad * 2);
  L.dzpart = take(BH * nq * kDPad * 4);
  L.dhtot = take(BH * kDPad * kDPad * 4);
  L.dztot = take(BH * kDPad * 4);
  L.dh16 = take(BH * kDPad * kDPad * 2);
  L.tau = take(BH * 4);
  L.total = off;
  return L;
}

bool bwd_tc_eligible(const sla_shape& s) { return s.in_dtype == SLA_BF16 && s.d == kDPad && s.bq == 128; }

cudaError_t launch_backward_tc(const sla_shape& s, const void* q, const void* k, const void* v, const void* dout,
                               const int32_t* kept, int k_keep, const float* alpha, int phi, float* dq, float* dk,
                               float* dv, float* dalpha, char* ws, cudaStream_t st) {
  const BwdTcLayout L = bwd_tc_layout(s);
  const int BH = s.B * s.H;
  const int nq = ceil_div(s.N, s.bq), nkv = ceil_div(s.N, s.bkv);
  cudaError_t e;
  // 1. sla_prepare, then the attention kernel with the statistics epilogue
  if ((e = launch_prepare(s, k, v, phi, L.fwd, ws, st)) != cudaSuccess) return e;
  {
    SparseArgs fa{};
    static const int32_t kNoBlocks = 0;
    fa.crit_idx = kept ? kept : &kNoBlocks;
    fa.negl_idx = nullptr;
    fa.list_stride = k_keep;
    fa.crit_max = k_keep;
    fa.negl_max = 0;
    fa.counts = nullptr;
    fa.alpha = alpha;
    fa.wproj = nullptr;
    fa.out = nullptr;
    fa.out_bf16 = 0;
    fa.bwd_do = dout;
    fa.bwd_rows = reinterpret_cast<float*>(ws + L.rows);
    fa.fp8 = 0;
    fa.wait_ns = kWaitLimitNs;
    fa.nb128 = ceil_div(s.N, 128);
    fa.BH = BH;
    fa.N = s.N;
    fa.d = s.d;
    fa.bq = s.bq;
    fa.nq = nq;
    fa.nkv = nkv;
    fa.sl2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(s.d)));
    fa.sigma = reinterpret_cast<const float*>(ws + L.fwd.sigma);
    fa.zblk = reinterpret_cast<const float*>(ws + L.fwd.zblk);
    fa.ztot = reinterpret_cast<const float*>(ws + L.fwd.ztot);
    fa.phi = phi;
    fa.status = reinterpret_cast<int*>(ws + L.fwd.status);
    fa.qsrc = q;
    if ((e = launch_sparse(fa, q, k, ws + L.fwd.phik, ws + L.fwd.v16, ws + L.fwd.hs16, nullptr, nullptr, nullptr,
                           st)) != cudaSuccess)
      return e;
  }
  const long long rows = static_cast<long long>(BH) * s.N;
  __half* phiq = reinterpret_cast<__half*>(ws + L.phiq);
  qphi_kernel<<<static_cast<unsigned>((rows * 16 + 255) / 256), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(q), phiq, rows, phi);
  int32_t* inv = reinterpret_cast<int32_t*>(ws + L.inv);
  int32_t* inv_n = reinterpret_cast<int32_t*>(ws + L.inv_n);
  if (k_keep > 0) {
    inv_lists_kernel<<<dim3((nkv + 7) / 8, BH), 256, 0, st>>>(kept, nq, nkv, k_keep, inv, inv_n);
  } else if ((e = cudaMemsetAsync(inv_n, 0, static_cast<size_t>(BH) * nkv * 4, st)) != cudaSuccess) {
    return e;
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  CUtensorMap mq, mdo, mk, mv, mpk, mh, mpq;
  using CU = CUtensorMapDataType;
  const CU BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, F16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if ((e = encode_map(&mq, q, BF, s.N, BH, 128)) != cudaSuccess) return e;
  if ((e = encode_map(&mdo, dout, BF, s.N, BH, 128)) != cudaSuccess) return e;
  if ((e = encode_map(&mk, k, BF, s.N, BH, 64)) != cudaSuccess) return e;
  if ((e = encode_map(&mv, v, BF, s.N, BH, 64)) != cudaSuccess) return e;
  if ((e = encode_map(&mpk, ws + L.fwd.phik, F16, s.N, BH, 64)) != cudaSuccess) return e;
  if ((e = encode_map(&mh, ws + L.fwd.hs16, F16, kDPad, BH, 128)) != cudaSuccess) return e;
  if ((e = encode_map(&mpq, phiq, F16, s.N, BH, 128)) != cudaSuccess) return e;

  TcArgs a{};
  a.BH = BH;
  a.N = s.N;
  a.nq = nq;
  a.nkv = nkv;
  a.kk = k_keep;
  a.phi = phi;
  a.sl2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(s.d)));
  a.scale = 1.0f / sqrtf(static_cast<float>(s.d));
  a.kept = kept;
  a.alpha = alpha;
  a.rows = reinterpret_cast<const float*>(ws + L.rows);
  a.sigma = reinterpret_cast<const float*>(ws + L.fwd.sigma);
  a.ztot = reinterpret_cast<const float*>(ws + L.fwd.ztot);
  a.inv = inv;
  a.inv_n = inv_n;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dhpart = reinterpret_cast<__half*>(ws + L.dhpart);
  a.dzpart = reinterpret_cast<float*>(ws + L.dzpart);
  a.status = reinterpret_cast<int*>(ws + L.fwd.status);
  a.wait_ns = kWaitLimitNs;
  float* dhtot = reinterpret_cast<float*>(ws + L.dhtot);
  float* dztot = reinterpret_cast<float*>(ws + L.dztot);
  __half* dh16 = reinterpret_cast<__half*>(ws + L.dh16);
  float* tau = reinterpret_cast<float*>(ws + L.tau);
  a.dztot = dztot;
  a.tau = tau;

  // 2. dQ per query tile; the tiles' -sigma dH_i (fp16) and dZ_i
  if ((e = cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dq::SMEM)) != cudaSuccess)
    return e;
  bwd_dq_kernel<<<static_cast<unsigned>(BH * nq), kTcThreads, dq::SMEM, st>>>(mq, mdo, mk, mv, mpk, mh, mpq, a);
  // 3. dH_tot, dZ_tot (tile order), tau dH_tot in fp16; dalpha
  dh_reduce_kernel<<<dim3(kDPad * kDPad / 256, BH), 256, 0, st>>>(a.dhpart, a.dzpart, a.sigma, nq, dhtot, dztot);
  dh_pack_kernel<<<BH, 256, 0, st>>>(dhtot, dh16, tau);
  const long long ntile = static_cast<long long>(BH) * nq;
  dalpha_kernel<<<static_cast<unsigned>((ntile * 32 + 255) / 256), 256, 0, st>>>(a.rows, s.N, nq, ntile, dalpha);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 4. dK, dV per key block: the sparse shares over the tiles keeping it, the linear
  //    shares from the totals minus those tiles' partials
  CUtensorMap mv16, mdhi, mdh;
  if ((e = encode_map(&mv16, ws + L.fwd.v16, F16, s.N, BH, 64)) != cudaSuccess) return e;
  if ((e = encode_map(&mdhi, a.dhpart, F16, kDPad, BH * nq, 128)) != cudaSuccess) return e;
  if ((e = encode_map(&mdh, dh16, F16, kDPad, BH, 128)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dkv::SMEM)) !=
      cudaSuccess)
    return e;
  bwd_dkv_kernel<<<static_cast<unsigned>(BH * nkv), kTcThreads, dkv::SMEM, st>>>(mq, mdo, mk, mv, mv16, mpk, mdhi,
                                                                                  mdh, a);
  return cudaGetLastError();
}

}  // namespace sla
