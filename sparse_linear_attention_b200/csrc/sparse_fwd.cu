// sparse_fwd.cu -- the attention kernel: block-sparse online-softmax branch,
// linear branch and the combine, for one 128-row query tile per CTA.
//
// Follows "SLA2 深度解读 …" (jefxiong.cn) §04 (O = alpha ⊙ O_s + (1-alpha) ⊙ O_l,
// both branches row-normalised), §08 (only mask-hit blocks run QK^T and PV
// in a FlashAttention-style online softmax; the missed blocks are handled by
// phi(Q) times the aggregated (K^phi)^T V; alpha per query block) and
// "SLA: Beyond Sparsity in Diffusion Transformers …" (papernotes.org)
// 关键设计 3 (H_i, Z_i, O_l = phi(Q_i) H_i / (phi(Q_i) Z_i), O = O_s + Proj(O_l))
// and 关键设计 4 (sparse and linear parts in one kernel; h_j added per block).
//
// B200 design (one CTA per (b,h, query block), 192 threads):
//   warp 4      TMA producer: Q tile once, then per listed key block its
//               K (bf16), phi(K) and V (fp16) tiles into a 3-stage ring.
//   warp 5      tcgen05 issuer (one thread):
//                 S_j   = Q K_j^T                    (bf16, 128x64, TMEM)
//                 H_ex += phi(K_j)^T V_j, Z_ex += phi(K_j)^T 1   (fp16)
//                 O    += P_j V_j                    (fp16 P from smem)
//               and, in the epilogue, phi(Q) H_i (bf16 hi + lo split) and for
//               SLA O_l W_proj (bf16 hi + lo).
//   warps 0..3  one query row per thread (TMEM lane = row): online softmax
//               with the running max refreshed only when it grows by more
//               than 2^8 (exact: the same stale max scales numerator and
//               denominator), P rounded to fp16, then the epilogue.
// The linear branch uses H_i = H_tot - sum over the listed blocks of
// phi(K_j)^T V_j (H_tot from sla_prepare), so a query block costs one extra
// 128x128x64 MMA per kept block instead of a sum over all unselected blocks.
// SLA's negligible blocks are listed too (H/Z only, no softmax).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "sla_device.cuh"
#include "sla_internal.h"
#include "sla_kernels.h"

namespace sla {

namespace {

constexpr int kThreads = 192;
constexpr int kStages = 3;
constexpr uint32_t OFF_Q = 0;                                   // Q tile, later phi(Q): 2 x [128 rows][128 B]
constexpr uint32_t STAGE_BYTES = 49152;                         // K | phi(K) | V, each 2 x [64 rows][128 B]
constexpr uint32_t OFF_ST = 32768;
constexpr uint32_t OFF_P = OFF_ST + kStages * STAGE_BYTES;      // 180224: 2 x [128 rows][128 B] fp16 P
constexpr uint32_t OFF_ONES = OFF_P + 2 * 16384;                // 212992: ones column for Z
constexpr uint32_t OFF_BAR = OFF_ONES + 2048;                   // 215040
constexpr uint32_t OFF_MISC = OFF_BAR + 256;                    // tmem base, abort flag
constexpr uint32_t OFF_Z = OFF_MISC + 64;                       // Z_i, 128 floats
constexpr uint32_t SMEM_BYTES = OFF_Z + 512 + 1024;             // + alignment slack
// epilogue reuse of the stage ring and P buffers
constexpr uint32_t OFF_HHI = OFF_ST;            // H_i hi, bf16, MN-major: 2 x [128 e][128 B]
constexpr uint32_t OFF_HLO = OFF_ST + 32768;    // H_i lo
constexpr uint32_t OFF_OLHI = OFF_ST + 65536;   // O_l hi, bf16, K-major like Q (SLA)
constexpr uint32_t OFF_OLLO = OFF_ST + 98304;   // O_l lo
constexpr uint32_t OFF_WP = OFF_P;              // W_proj, bf16, MN-major (SLA)
static_assert(OFF_OLLO + 32768 <= OFF_P, "epilogue buffers overlap P");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns (512 allocated; one CTA per SM)
constexpr uint32_t T_S0 = 0, T_S1 = 64, T_O = 128, T_HK = 256, T_ZK = 384;
constexpr uint32_t T_NUM = 0;    // epilogue: reuses the S buffers
constexpr uint32_t T_PROJ = 256; // SLA epilogue: reuses H_ex after it is read
constexpr uint32_t TMEM_COLS = 512;

enum {
  B_QFULL = 0,
  B_KVFULL = 1,   // +stage
  B_KVEMPTY = 4,  // +stage
  B_SFULL = 7,    // +buffer
  B_PFULL = 9,    // +buffer
  B_PEMPTY = 11,  // +buffer
  B_OFINAL = 13,
  B_EPI = 14,
  B_NUM = 15,
  B_PROJR = 16,
  B_PROJF = 17,
  B_DRAIN = 18,
  NBAR = 19
};

// Warp-uniform bounded wait: every lane polls, the warp agrees on the verdict.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok) != 0;
}

__device__ __forceinline__ int block_at(const int32_t* crit, const int32_t* negl, int n_crit, int it, int nkv,
                                        int* status) {
  int j = it < n_crit ? crit[it] : negl[it - n_crit];
  if (j < 0 || j >= nkv) {
    report_error(status, SLA_ERR_DEVICE_INDEX);
    j = 0;
  }
  return j;
}

__global__ void __launch_bounds__(kThreads, 1)
    sparse_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmPhi, const __grid_constant__ CUtensorMap tmV,
                      const SparseArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  float* zsh = reinterpret_cast<float*>(sm + OFF_Z);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qb = blockIdx.x % a.nq;
  const int bh = blockIdx.x / a.nq;
  const long long row = static_cast<long long>(bh) * a.nq + qb;

  int n_crit = a.crit_max, n_negl = 0;
  if (a.counts) {
    n_crit = a.counts[2 * row];
    n_negl = a.counts[2 * row + 1];
  }
  if (n_crit < 0 || n_crit > a.crit_max || n_negl < 0 || n_negl > a.negl_max || n_crit + n_negl > a.nkv) {
    if (tid == 0) report_error(a.status, SLA_ERR_DEVICE_INDEX);
    n_crit = 0;
    n_negl = 0;
  }
  const int32_t* crit = a.crit_idx + row * a.list_stride;
  const int32_t* negl = a.negl_idx ? a.negl_idx + row * a.list_stride : crit;
  const int n_total = n_crit + n_negl;
  const bool has_lin = (a.nkv - n_total) > 0;

  // ---------------------------------------------------------------- set-up
  for (int i = tid; i < 2048 / 4; i += kThreads)
    reinterpret_cast<uint32_t*>(sm + OFF_ONES)[i] = (i < 32) ? 0x3C003C00u : 0u;  // fp16 ones in row 0
  if (tid == 0) {
    mbar_init(&bars[B_QFULL], 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[B_KVFULL + s], 1);
      mbar_init(&bars[B_KVEMPTY + s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[B_SFULL + b], 1);
      mbar_init(&bars[B_PFULL + b], 128);
      mbar_init(&bars[B_PEMPTY + b], 1);
    }
    mbar_init(&bars[B_OFINAL], 1);
    mbar_init(&bars[B_EPI], 128);
    mbar_init(&bars[B_NUM], 1);
    mbar_init(&bars[B_PROJR], 128);
    mbar_init(&bars[B_PROJF], 1);
    mbar_init(&bars[B_DRAIN], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmPhi);
      tma_prefetch_desc(&tmV);
      const int qrow0 = qb * a.bq;
      mbar_arrive_expect_tx(&bars[B_QFULL], 32768);
      tma_load_3d(sm + OFF_Q, &tmQ, &bars[B_QFULL], 0, qrow0, bh);
      tma_load_3d(sm + OFF_Q + 16384, &tmQ, &bars[B_QFULL], 64, qrow0, bh);
      int issued = 0;
      for (int it = 0; it < n_total; ++it) {
        const int st = it % kStages;
        if (it >= kStages && !mbar_wait(&bars[B_KVEMPTY + st], ((it / kStages) - 1) & 1, abort_flag, a.status))
          break;
        const int j = block_at(crit, negl, n_crit, it, a.nkv, a.status);
        const bool isc = it < n_crit;
        uint8_t* sb = sm + OFF_ST + st * STAGE_BYTES;
        uint64_t* fb = &bars[B_KVFULL + st];
        mbar_arrive_expect_tx(fb, isc ? 49152u : 32768u);
        const int krow = j * kBlockKV;
        if (isc) {
          tma_load_3d(sb, &tmK, fb, 0, krow, bh);
          tma_load_3d(sb + 8192, &tmK, fb, 64, krow, bh);
        }
        tma_load_3d(sb + 16384, &tmPhi, fb, 0, krow, bh);
        tma_load_3d(sb + 16384 + 8192, &tmPhi, fb, 64, krow, bh);
        tma_load_3d(sb + 32768, &tmV, fb, 0, krow, bh);
        tma_load_3d(sb + 32768 + 8192, &tmV, fb, 64, krow, bh);
        issued = it + 1;
      }
      // every issued copy must land before the CTA may exit
      mbar_wait_drain(&bars[B_QFULL], 0);
      for (int it = issued > kStages ? issued - kStages : 0; it < issued; ++it)
        mbar_wait_drain(&bars[B_KVFULL + it % kStages], (it / kStages) & 1);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = idesc_f16(1, 0, 0, 128, 64);   // Q (K-major) x K_j (K-major), bf16
      const uint32_t id_h = idesc_f16(0, 1, 1, 128, 128);   // phi(K)^T (MN-major) x V (MN-major), f16
      const uint32_t id_z = idesc_f16(0, 1, 0, 128, 16);    // phi(K)^T x ones (K-major), f16
      const uint32_t id_pv = idesc_f16(0, 0, 1, 128, 128);  // P (K-major) x V (MN-major), f16
      const uint32_t id_bf = idesc_f16(1, 0, 1, 128, 128);  // K-major x MN-major, bf16
      const uint32_t sQ = smem_u32(sm + OFF_Q), sST = smem_u32(sm + OFF_ST), sP = smem_u32(sm + OFF_P);
      const uint32_t sOnes = smem_u32(sm + OFF_ONES);
      auto issue_qk = [&](int st, int b) {
        const uint32_t kb = sST + st * STAGE_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk & 3) * 32u;
          const uint64_t ad = sdesc_sw128(sQ + (kk >> 2) * 16384u + koff, 16, 1024);
          const uint64_t bd = sdesc_sw128(kb + (kk >> 2) * 8192u + koff, 16, 1024);
          mma_f16_ss(tmem + (b ? T_S1 : T_S0), ad, bd, id_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_h = [&](int st, bool first) {
        const uint32_t pb = sST + st * STAGE_BYTES + 16384, vb = sST + st * STAGE_BYTES + 32768;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = sdesc_sw128(pb + kk * 2048u, 8192, 1024);
          const uint64_t bd = sdesc_sw128(vb + kk * 2048u, 8192, 1024);
          const uint64_t od = sdesc_sw128(sOnes + kk * 32u, 16, 1024);
          const uint32_t acc = (first && kk == 0) ? 0u : 1u;
          mma_f16_ss(tmem + T_HK, ad, bd, id_h, acc);
          mma_f16_ss(tmem + T_ZK, ad, od, id_z, acc);
        }
      };
      auto issue_pv = [&](int st, int b, bool first) {
        const uint32_t vb = sST + st * STAGE_BYTES + 32768;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = sdesc_sw128(sP + b * 16384u + kk * 32u, 16, 1024);
          const uint64_t bd = sdesc_sw128(vb + kk * 2048u, 8192, 1024);
          mma_f16_ss(tmem + T_O, ad, bd, id_pv, (first && kk == 0) ? 0u : 1u);
        }
      };
      // A (K-major, Q-tile layout) x B (MN-major, [128 K-rows] x 2 chunks of 64 N) -> tmem col
      auto issue_bf = [&](uint32_t a_off, uint32_t b_off, uint32_t col, bool first) {
        const uint32_t ab = smem_u32(sm + a_off), bb = smem_u32(sm + b_off);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = sdesc_sw128(ab + (kk >> 2) * 16384u + (kk & 3) * 32u, 16, 1024);
          const uint64_t bd = sdesc_sw128(bb + kk * 2048u, 16384, 1024);
          mma_f16_ss(tmem + col, ad, bd, id_bf, (first && kk == 0) ? 0u : 1u);
        }
      };

      bool ok = mbar_wait(&bars[B_QFULL], 0, abort_flag, a.status);
      if (ok && n_crit > 0) {
        ok = mbar_wait(&bars[B_KVFULL + 0], 0, abort_flag, a.status);
        if (ok) {
          tc_fence_after();
          issue_qk(0, 0);
          mma_commit(&bars[B_SFULL + 0]);
        }
      }
      bool h_first = true;
      for (int it = 0; ok && it < n_crit; ++it) {
        const int st = it % kStages;
        if (it + 1 < n_crit) {
          const int st1 = (it + 1) % kStages;
          if (!mbar_wait(&bars[B_KVFULL + st1], ((it + 1) / kStages) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_qk(st1, (it + 1) & 1);
          mma_commit(&bars[B_SFULL + ((it + 1) & 1)]);
        }
        issue_h(st, h_first);
        h_first = false;
        if (!mbar_wait(&bars[B_PFULL + (it & 1)], (it >> 1) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv(st, it & 1, it == 0);
        mma_commit(&bars[B_PEMPTY + (it & 1)]);
        mma_commit(&bars[B_KVEMPTY + st]);
      }
      for (int it = n_crit; ok && it < n_total; ++it) {
        const int st = it % kStages;
        if (!mbar_wait(&bars[B_KVFULL + st], (it / kStages) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_h(st, h_first);
        h_first = false;
        mma_commit(&bars[B_KVEMPTY + st]);
      }
      if (ok) mma_commit(&bars[B_OFINAL]);
      if (ok && has_lin) {
        ok = mbar_wait(&bars[B_EPI], 0, abort_flag, a.status);
        if (ok) {
          tc_fence_after();
          issue_bf(OFF_Q, OFF_HHI, T_NUM, true);
          issue_bf(OFF_Q, OFF_HLO, T_NUM, false);
          mma_commit(&bars[B_NUM]);
        }
      }
      if (ok && has_lin && a.wproj != nullptr) {
        ok = mbar_wait(&bars[B_PROJR], 0, abort_flag, a.status);
        if (ok) {
          tc_fence_after();
          issue_bf(OFF_OLHI, OFF_WP, T_PROJ, true);
          issue_bf(OFF_OLLO, OFF_WP, T_PROJ, false);
          mma_commit(&bars[B_PROJF]);
        }
      }
      // all MMAs must finish before the CTA releases TMEM
      mma_commit(&bars[B_DRAIN]);
      mbar_wait_drain(&bars[B_DRAIN], 0);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int r = tid;  // query row of the tile = TMEM lane
    const uint32_t lrow = static_cast<uint32_t>(warp * 32) << 16;
    const int tok = qb * a.bq + r;
    const bool row_valid = (r < a.bq) && (tok < a.N);
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true, passed_nb = false;
    for (int it = 0; it < n_crit; ++it) {
      const int b = it & 1;
      if (!warp_wait(&bars[B_SFULL + b], (it >> 1) & 1, abort_flag, a.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[64];
      tmem_ld32(tmem + lrow + (b ? T_S1 : T_S0), s);
      tmem_ld32(tmem + lrow + (b ? T_S1 : T_S0) + 32, s + 32);
      tmem_wait_ld();
      const int j = block_at(crit, negl, n_crit, it, a.nkv, nullptr);
      const int nvalid = a.N - j * kBlockKV;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        if (c >= nvalid) s[c] = -INFINITY;
        mx = fmaxf(mx, s[c]);
      }
      const float mt = mx * a.sl2;
      const bool need = mt > m_run + 8.0f;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mt : m_run;
        const float f = need ? exp2f(m_run - m_new) : 1.0f;
        if (it > 0) {
          // O holds P V of the previous blocks: wait for the last PV, rescale
          if (!warp_wait(&bars[B_PEMPTY + ((it - 1) & 1)], ((it - 1) >> 1) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            float o[32];
            tmem_ld32(tmem + lrow + T_O + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= f;
            tmem_st32(tmem + lrow + T_O + cc * 32, o);
          }
          tmem_wait_st();
        }
        l_run *= f;
        m_run = m_new;
      }
      if (it >= 2 && !warp_wait(&bars[B_PEMPTY + b], ((it - 2) >> 1) & 1, abort_flag, a.status)) {
        ok = false;
        break;
      }
      uint8_t* prow = sm + OFF_P + b * 16384;
      const float nm = -m_run;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        uint32_t h[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = exp2f(fmaf(s[8 * u + 2 * e], a.sl2, nm));
          const float p1 = exp2f(fmaf(s[8 * u + 2 * e + 1], a.sl2, nm));
          h[e] = pack_half2(p0, p1);
          const float2 back = unpack_half2(h[e]);
          l_run += back.x + back.y;
        }
        *reinterpret_cast<uint4*>(prow + sw128_off(r, u)) = make_uint4(h[0], h[1], h[2], h[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[B_PFULL + b]);
    }

    if (ok) ok = warp_wait(&bars[B_OFINAL], 0, abort_flag, a.status);
    if (ok) tc_fence_after();
    float den = 0.0f;
    if (ok && has_lin) {
      // H_i = H_tot - H_ex (row e = r), split into bf16 hi + lo, MN-major
      const float* ht = a.htot + (static_cast<long long>(bh) * kDPad + r) * kDPad;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float hk[32];
        if (n_total > 0) {
          tmem_ld32(tmem + lrow + T_HK + cc * 32, hk);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) hk[i] = 0.0f;
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int c0 = cc * 32 + q4 * 8;
          const float4 t0 = *reinterpret_cast<const float4*>(ht + c0);
          const float4 t1 = *reinterpret_cast<const float4*>(ht + c0 + 4);
          const float dv[8] = {t0.x - hk[q4 * 8 + 0], t0.y - hk[q4 * 8 + 1], t0.z - hk[q4 * 8 + 2],
                               t0.w - hk[q4 * 8 + 3], t1.x - hk[q4 * 8 + 4], t1.y - hk[q4 * 8 + 5],
                               t1.z - hk[q4 * 8 + 6], t1.w - hk[q4 * 8 + 7]};
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            hi[e] = pack_bf162(dv[2 * e], dv[2 * e + 1]);
            const float2 hb = unpack_bf162(hi[e]);
            lo[e] = pack_bf162(dv[2 * e] - hb.x, dv[2 * e + 1] - hb.y);
          }
          const uint32_t off = (c0 >> 6) * 16384u + sw128_off(r, (c0 & 63) >> 3);
          *reinterpret_cast<uint4*>(sm + OFF_HHI + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(sm + OFF_HLO + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      float zk = 0.0f;
      if (n_total > 0) {
        float z[32];
        tmem_ld32(tmem + lrow + T_ZK, z);
        tmem_wait_ld();
        zk = z[0];
      }
      zsh[r] = a.ztot[static_cast<long long>(bh) * kDPad + r] - zk;

      // phi(Q) in place over the Q tile (bf16), channels past d zero
      float x[128];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const uint4 w = *reinterpret_cast<const uint4*>(sm + OFF_Q + (u >> 3) * 16384u + sw128_off(r, u & 7));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f2 = unpack_bf162(ww[e]);
          x[8 * u + 2 * e] = f2.x;
          x[8 * u + 2 * e + 1] = f2.y;
        }
      }
      if (a.phi == SLA_PHI_SOFTMAX) {
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c < a.d) mx = fmaxf(mx, x[c]);
        float sum = 0.0f;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          x[c] = c < a.d ? expf(x[c] - mx) : 0.0f;
          sum += x[c];
        }
        const float inv = 1.0f / sum;
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] *= inv;
      } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] = c < a.d ? elu1(x[c]) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        uint32_t h[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          h[e] = pack_bf162(x[8 * u + 2 * e], x[8 * u + 2 * e + 1]);
          const float2 back = unpack_bf162(h[e]);  // the denominator uses the rounded phi(Q)
          x[8 * u + 2 * e] = back.x;
          x[8 * u + 2 * e + 1] = back.y;
        }
        *reinterpret_cast<uint4*>(sm + OFF_Q + (u >> 3) * 16384u + sw128_off(r, u & 7)) =
            make_uint4(h[0], h[1], h[2], h[3]);
      }
      named_bar_sync(1, 128);  // Z_i complete
      passed_nb = true;
#pragma unroll
      for (int e = 0; e < 128; ++e) den += x[e] * zsh[e];
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[B_EPI]);
      ok = warp_wait(&bars[B_NUM], 0, abort_flag, a.status);
      if (ok) tc_fence_after();
    }

    if (ok) {
      const float inv_l = (n_crit > 0 && l_run > 0.0f) ? 1.0f / l_run : 0.0f;
      const float inv_den = (has_lin && den > 0.0f) ? 1.0f / den : 0.0f;
      const long long obase = (static_cast<long long>(bh) * a.N + tok) * a.d;
      if (a.wproj != nullptr && has_lin) {
        // SLA: O_l -> bf16 hi + lo (K-major), W_proj -> smem (MN-major), MMA
        const __nv_bfloat16* wp = static_cast<const __nv_bfloat16*>(a.wproj);
        for (int idx = r; idx < 128 * 16; idx += 128) {
          const int e = idx >> 4, u = idx & 15;
          uint4 w = make_uint4(0, 0, 0, 0);
          if (e < a.d && 8 * u < a.d) w = *reinterpret_cast<const uint4*>(wp + e * a.d + 8 * u);
          *reinterpret_cast<uint4*>(sm + OFF_WP + (u >> 3) * 16384u + sw128_off(e, u & 7)) = w;
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float nmv[32];
          tmem_ld32(tmem + lrow + T_NUM + cc * 32, nmv);
          tmem_wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int c0 = cc * 32 + q4 * 8;
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float v0 = nmv[q4 * 8 + 2 * e] * inv_den, v1 = nmv[q4 * 8 + 2 * e + 1] * inv_den;
              hi[e] = pack_bf162(v0, v1);
              const float2 hb = unpack_bf162(hi[e]);
              lo[e] = pack_bf162(v0 - hb.x, v1 - hb.y);
            }
            const uint32_t off = (c0 >> 6) * 16384u + sw128_off(r, (c0 & 63) >> 3);
            *reinterpret_cast<uint4*>(sm + OFF_OLHI + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(sm + OFF_OLLO + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars[B_PROJR]);
        ok = warp_wait(&bars[B_PROJF], 0, abort_flag, a.status);
        if (ok) tc_fence_after();
      }
      if (ok) {
        const float al = a.alpha ? a.alpha[row] : 1.0f;
        const float w_s = a.wproj ? inv_l : al * inv_l;
        const float w_l = a.wproj ? 1.0f : (1.0f - al) * inv_den;
        const uint32_t lin_col = a.wproj ? T_PROJ : T_NUM;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float o[32], nmv[32];
          if (n_crit > 0) {
            tmem_ld32(tmem + lrow + T_O + cc * 32, o);
          }
          if (has_lin) {
            tmem_ld32(tmem + lrow + lin_col + cc * 32, nmv);
          }
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float os = n_crit > 0 ? o[i] * w_s : 0.0f;
            const float ol = has_lin ? nmv[i] * w_l : 0.0f;
            o[i] = os + ol;
          }
          if (row_valid) {
            if (a.out_bf16) {
              __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + obase;
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const int c0 = cc * 32 + q4 * 8;
                if (c0 < a.d)
                  *reinterpret_cast<uint4*>(dst + c0) =
                      make_uint4(pack_bf162(o[q4 * 8], o[q4 * 8 + 1]), pack_bf162(o[q4 * 8 + 2], o[q4 * 8 + 3]),
                                 pack_bf162(o[q4 * 8 + 4], o[q4 * 8 + 5]), pack_bf162(o[q4 * 8 + 6], o[q4 * 8 + 7]));
              }
            } else {
              float* dst = static_cast<float*>(a.out) + obase;
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4) {
                const int c0 = cc * 32 + q4 * 4;
                if (c0 < a.d)
                  *reinterpret_cast<float4*>(dst + c0) = make_float4(o[q4 * 4], o[q4 * 4 + 1], o[q4 * 4 + 2], o[q4 * 4 + 3]);
              }
            }
          }
        }
      }
    }
    // a warp that gave up before the named barrier still releases the others
    if (has_lin && !passed_nb) asm volatile("bar.arrive 1, 128;" ::: "memory");
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_sparse(const SparseArgs& a, const void* q_bf16_128, const void* k_bf16_128,
                          const void* phik16, const void* v16, cudaStream_t st) {
  CUtensorMap mq, mk, mp, mv;
  cudaError_t e;
  if ((e = encode_map(&mq, q_bf16_128, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.N, a.BH, 128)) != cudaSuccess) return e;
  if ((e = encode_map(&mk, k_bf16_128, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.N, a.BH, 64)) != cudaSuccess) return e;
  if ((e = encode_map(&mp, phik16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.N, a.BH, 64)) != cudaSuccess) return e;
  if ((e = encode_map(&mv, v16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.N, a.BH, 64)) != cudaSuccess) return e;
  e = cudaFuncSetAttribute(sparse_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(a.BH) * a.nq;
  sparse_fwd_kernel<<<static_cast<unsigned>(grid), kThreads, SMEM_BYTES, st>>>(mq, mk, mp, mv, a);
  return cudaGetLastError();
}

}  // namespace sla
