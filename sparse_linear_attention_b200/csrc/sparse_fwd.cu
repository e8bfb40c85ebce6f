// sparse_fwd.cu -- the attention kernel: block-sparse online-softmax branch,
// linear branch and the combine.
//
// Follows "SLA2 深度解读 …" (jefxiong.cn) §04 (O = alpha ⊙ O_s + (1-alpha) ⊙ O_l,
// both branches row-normalised), §08 (only mask-hit blocks run QK^T and PV
// in a FlashAttention-style online softmax; the missed blocks are handled by
// phi(Q) times the aggregated (K^phi)^T V; alpha per query block) and
// "SLA: Beyond Sparsity in Diffusion Transformers …" (papernotes.org)
// 关键设计 3 (H_i, Z_i, O_l = phi(Q_i) H_i / (phi(Q_i) Z_i), O = O_s + Proj(O_l))
// and 关键设计 4 (sparse and linear parts in one kernel; h_j added per block).
//
// B200 design: persistent CTAs (one per SM), each walking 128-row query tiles
// (b, h, query block) in head-major order; 320 threads:
//   warp 8      TMA producer, running ahead across tiles: per listed key
//               block its K tile (bf16) into a 3-slot ring that frees as soon
//               as the S MMA has read it, and its phi(K), V tiles (fp16) into a
//               3-slot ring that frees after PV; per tile the Q tile and the
//               fp16 H_tot / sigma tile of its head.
//   warp 9      tcgen05 issuer (one thread), fp32 accumulators in TMEM:
//                 S_j   = Q K_j^T                    (bf16 operands from smem)
//                 H_ex += phi(K_j)^T V_j                (fp16)
//                 O    += P_j V_j                    (fp16 P read from TMEM)
//               and per tile phi(Q) H_i (fp16, phi(Q) in TMEM), for SLA also
//               O_l W_proj (bf16 hi + lo split, O_l in TMEM).
//   warps 0..7  softmax and epilogue: warp w owns query rows 32(w%4)..+31
//               (its TMEM lane quarter) and key / channel half w/4, so two
//               warps share each row and every sub-partition runs two.
//               Online softmax in log2 units with the running max refreshed
//               only when a block's max exceeds it by more than 15 (exact:
//               the stale max scales numerator and denominator alike, and
//               p <= 2^15 still fits fp16); P is rounded to fp16 and stored
//               to TMEM for the PV MMA.
// The linear branch uses H_i = H_tot - sum over the listed blocks of
// phi(K_j)^T V_j (H_tot from sla_prepare): one extra 128x128x64 MMA per
// listed block instead of a sum over every unselected block; Z_ex sums the
// per-block column sums of phi(K) that sla_prepare stores.  H_i enters the
// MMA as fp16 scaled by an exact power of two sigma >= max_e Z_tot[e], which
// bounds |H_i / sigma| by max|V|; H_tot / sigma arrives by TMA and the
// epilogue subtracts H_ex / sigma in place.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "sla_device.cuh"
#include "sla_internal.h"
#include "sla_kernels.h"

namespace sla {

namespace {

constexpr int kThreads = 320;
constexpr int kCompute = 256;
constexpr int kStages = 3;  // slots of each ring

// Shared-memory layout.  bf16 branch: Q tile 2 x [128 rows][128 B], K tile
// 2 x [64 rows][128 B], V slot = phi(K) | V (fp16, each 2 x [64 rows][128 B]).
// e4m3 branch: Q8 [128 rows][128 B], K8 [64 rows][128 B], V slot = phi(K) |
// V (fp16) | V8 [64 rows][128 B].  Then H_i / W_proj (MN-major, 32 KB),
// barriers, flags, exchange buffers.
template <bool kFP8>
struct Lay {
  static constexpr uint32_t QBYTES = kFP8 ? 16384 : 32768;
  static constexpr uint32_t KSLOT = kFP8 ? 8192 : 16384;
  static constexpr uint32_t VSLOT = kFP8 ? 40960 : 32768;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = QBYTES;
  static constexpr uint32_t OFF_V = OFF_K + kStages * KSLOT;
  static constexpr uint32_t OFF_H = OFF_V + kStages * VSLOT;
  static constexpr uint32_t OFF_BAR = OFF_H + 32768;
  static constexpr uint32_t OFF_MISC = OFF_BAR + 256;  // tmem base, abort flag
  static constexpr uint32_t OFF_RED = OFF_MISC + 64;   // [4 slots][2 halves][128 rows] floats
  static constexpr uint32_t OFF_Z = OFF_RED + 4096;    // Z_i [128] + Z_ex halves [2][128] floats
  static constexpr uint32_t SMEM_BYTES = OFF_Z + 1536 + 1024;  // + alignment slack
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && OFF_H % 1024 == 0, "1 KB aligned tiles");
};

// TMEM columns (512 allocated; one CTA per SM)
constexpr uint32_t T_S0 = 0, T_S1 = 64, T_P0 = 128, T_P1 = 160, T_O = 192, T_HK = 320;
constexpr uint32_t T_PHIQ = 0;    // epilogue: phi(Q) as the A operand (fp16 pairs), 64 columns
constexpr uint32_t T_NUM = 64;    // epilogue: phi(Q) H_i, 128 columns
constexpr uint32_t T_OLHI = 64;   // SLA epilogue: O_l hi / lo (bf16 pairs), 64 columns each
constexpr uint32_t T_OLLO = 128;
constexpr uint32_t T_PROJ = 320;  // SLA epilogue: O_l W_proj
constexpr uint32_t TMEM_COLS = 512;

enum {
  B_QFULL = 0,
  B_QFREE = 1,
  B_KFULL = 2,    // +slot
  B_KEMPTY = 5,   // +slot
  B_VFULL = 8,    // +slot
  B_VEMPTY = 11,  // +slot
  B_SFULL = 14,   // +buffer
  B_PFULL = 16,   // +buffer
  B_PEMPTY = 18,  // +buffer
  B_HFULL = 20,
  B_OFINAL = 21,
  B_EPI = 22,
  B_NUM = 23,
  B_EPIDONE = 24,
  B_PROJR = 25,
  B_PROJF = 26,
  B_DRAIN = 27,
  NBAR = 28
};
static_assert(NBAR * 8 <= 256, "barrier area");

struct Tile {
  int bh, qb;
  long long row;
  int n_crit, n_negl, n_total;
  const int32_t* crit;
  const int32_t* negl;
  bool has_lin;
};

__device__ __forceinline__ Tile tile_at(const SparseArgs& a, int t, bool report) {
  Tile T;
  T.qb = t % a.nq;
  T.bh = t / a.nq;
  T.row = static_cast<long long>(T.bh) * a.nq + T.qb;
  T.n_crit = a.crit_max;
  T.n_negl = 0;
  if (a.counts) {
    T.n_crit = a.counts[2 * T.row];
    T.n_negl = a.counts[2 * T.row + 1];
  }
  if (T.n_crit < 0 || T.n_crit > a.crit_max || T.n_negl < 0 || T.n_negl > a.negl_max ||
      T.n_crit + T.n_negl > a.nkv) {
    if (report) report_error(a.status, SLA_ERR_DEVICE_INDEX);
    T.n_crit = 0;
    T.n_negl = 0;
  }
  T.n_total = T.n_crit + T.n_negl;
  T.crit = a.crit_idx + T.row * a.list_stride;
  T.negl = a.negl_idx ? a.negl_idx + T.row * a.list_stride : T.crit;
  T.has_lin = (a.nkv - T.n_total) > 0;
  return T;
}

__device__ __forceinline__ int block_at(const Tile& T, int it, int nkv, int* status) {
  int j = it < T.n_crit ? T.crit[it] : T.negl[it - T.n_crit];
  if (j < 0 || j >= nkv) {
    report_error(status, SLA_ERR_DEVICE_INDEX);
    j = 0;
  }
  return j;
}

// Warp-uniform bounded wait: every lane polls, the warp agrees on the verdict.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok) != 0;
}

template <bool kFP8>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmPhi, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmV8,
                      const SparseArgs a) {
  using L = Lay<kFP8>;
  constexpr uint32_t OFF_Q = L::OFF_Q, OFF_K = L::OFF_K, OFF_V = L::OFF_V, OFF_H = L::OFF_H;
  constexpr uint32_t OFF_BAR = L::OFF_BAR, OFF_MISC = L::OFF_MISC, OFF_RED = L::OFF_RED, OFF_Z = L::OFF_Z;
  constexpr uint32_t KSLOT = L::KSLOT, VSLOT = L::VSLOT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(sm + OFF_RED);
  float* zsh = reinterpret_cast<float*>(sm + OFF_Z);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles = a.BH * a.nq;

  // ---------------------------------------------------------------- set-up
  if (tid == 0) {
    mbar_init(&bars[B_QFULL], 1);
    mbar_init(&bars[B_QFREE], kCompute);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[B_KFULL + s], 1);
      mbar_init(&bars[B_KEMPTY + s], 1);
      mbar_init(&bars[B_VFULL + s], 1);
      mbar_init(&bars[B_VEMPTY + s], 1);
    }
    mbar_init(&bars[B_HFULL], 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[B_SFULL + b], 1);
      mbar_init(&bars[B_PFULL + b], kCompute);
      mbar_init(&bars[B_PEMPTY + b], 1);
    }
    mbar_init(&bars[B_OFINAL], 1);
    mbar_init(&bars[B_EPI], kCompute);
    mbar_init(&bars[B_NUM], 1);
    mbar_init(&bars[B_EPIDONE], kCompute);
    mbar_init(&bars[B_PROJR], kCompute);
    mbar_init(&bars[B_PROJF], 1);
    mbar_init(&bars[B_DRAIN], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmPhi);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmH);
      if constexpr (kFP8) tma_prefetch_desc(&tmV8);
      int gk = 0, gv = 0, q_issued = 0, h_issued = 0;
      bool ok = true;
      auto load_block = [&](const Tile& T, int it) -> bool {
        const int j = block_at(T, it, a.nkv, a.status);
        const int krow = j * kBlockKV;
        if (it < T.n_crit) {
          const int sl = gk % kStages;
          if (gk >= kStages && !mbar_wait(&bars[B_KEMPTY + sl], ((gk / kStages) - 1) & 1, abort_flag, a.status))
            return false;
          uint64_t* fb = &bars[B_KFULL + sl];
          mbar_arrive_expect_tx(fb, KSLOT);
          tma_load_3d(sm + OFF_K + sl * KSLOT, &tmK, fb, 0, krow, T.bh);
          if constexpr (!kFP8) tma_load_3d(sm + OFF_K + sl * KSLOT + 8192, &tmK, fb, 64, krow, T.bh);
          ++gk;
        }
        const int sl = gv % kStages;
        if (gv >= kStages && !mbar_wait(&bars[B_VEMPTY + sl], ((gv / kStages) - 1) & 1, abort_flag, a.status))
          return false;
        uint8_t* vb = sm + OFF_V + sl * VSLOT;
        uint64_t* fb = &bars[B_VFULL + sl];
        mbar_arrive_expect_tx(fb, VSLOT);
        tma_load_3d(vb, &tmPhi, fb, 0, krow, T.bh);
        tma_load_3d(vb + 8192, &tmPhi, fb, 64, krow, T.bh);
        tma_load_3d(vb + 16384, &tmV, fb, 0, krow, T.bh);
        tma_load_3d(vb + 16384 + 8192, &tmV, fb, 64, krow, T.bh);
        if constexpr (kFP8) tma_load_3d(vb + 32768, &tmV8, fb, 0, krow, T.bh);
        ++gv;
        return true;
      };
      int ti = 0;
      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++ti) {
        const Tile T = tile_at(a, t, true);
        const int pre = T.n_total < kStages ? T.n_total : kStages;
        int it = 0;
        for (; ok && it < pre; ++it) ok = load_block(T, it);  // key blocks first: they only need ring slots
        if (!ok) break;
        if (ti > 0 && !mbar_wait(&bars[B_QFREE], (ti - 1) & 1, abort_flag, a.status)) break;
        mbar_arrive_expect_tx(&bars[B_QFULL], L::QBYTES);
        tma_load_3d(sm + OFF_Q, &tmQ, &bars[B_QFULL], 0, T.qb * a.bq, T.bh);
        if constexpr (!kFP8) tma_load_3d(sm + OFF_Q + 16384, &tmQ, &bars[B_QFULL], 64, T.qb * a.bq, T.bh);
        q_issued = ti + 1;
        if (T.has_lin) {
          // H_tot / sigma of this head into the H buffer once the previous tile is done with it
          if (ti > 0 && !mbar_wait(&bars[B_EPIDONE], (ti - 1) & 1, abort_flag, a.status)) break;
          mbar_arrive_expect_tx(&bars[B_HFULL], 32768);
          tma_load_3d(sm + OFF_H, &tmH, &bars[B_HFULL], 0, 0, T.bh);
          tma_load_3d(sm + OFF_H + 16384, &tmH, &bars[B_HFULL], 64, 0, T.bh);
          ++h_issued;
        }
        for (; ok && it < T.n_total; ++it) ok = load_block(T, it);
      }
      // every issued copy must land before the CTA may exit
      if (q_issued > 0) mbar_wait_drain(&bars[B_QFULL], (q_issued - 1) & 1);
      if (h_issued > 0) mbar_wait_drain(&bars[B_HFULL], (h_issued - 1) & 1);
      for (int g = gk > kStages ? gk - kStages : 0; g < gk; ++g)
        mbar_wait_drain(&bars[B_KFULL + g % kStages], (g / kStages) & 1);
      for (int g = gv > kStages ? gv - kStages : 0; g < gv; ++g)
        mbar_wait_drain(&bars[B_VFULL + g % kStages], (g / kStages) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = idesc_f16(1, 0, 0, 128, 64);   // Q (K-major) x K_j (K-major), bf16
      const uint32_t id_h = idesc_f16(0, 1, 1, 128, 128);   // phi(K)^T (MN-major) x V (MN-major), f16
      const uint32_t id_pv = idesc_f16(0, 0, 1, 128, 128);  // P (TMEM) x V (MN-major), f16
      const uint32_t id_bf = idesc_f16(1, 0, 1, 128, 128);  // TMEM A x MN-major B, bf16
      // Descriptors built once; a byte offset d inside a tile adds d >> 4 to the
      // start-address field (addresses stay below 2^18, so the field cannot carry).
      const uint64_t dQ = sdesc_sw128(smem_u32(sm + OFF_Q), 16, 1024);
      const uint64_t dK = sdesc_sw128(smem_u32(sm + OFF_K), 16, 1024);
      const uint64_t dPhi = sdesc_sw128(smem_u32(sm + OFF_V), 8192, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(sm + OFF_V) + 16384, 8192, 1024);
      const uint64_t dH = sdesc_sw128(smem_u32(sm + OFF_H), 16384, 1024);
      const uint64_t dV8 = sdesc_sw128(smem_u32(sm + OFF_V) + 32768, 16, 1024);  // MN-major, N fits one atom
      const uint32_t id_qk8 = idesc_f8(0, 0, 128, 64);   // Q8 (K-major) x K8 (K-major), e4m3
      const uint32_t id_pv8 = idesc_f8(0, 1, 128, 128);  // P8 (TMEM) x V8 (MN-major), e4m3
      auto issue_qk = [&](int sl, int b) {
        const uint64_t kb = dK + ((sl * KSLOT) >> 4);
        const uint32_t d = tmem + (b ? T_S1 : T_S0);
        if constexpr (kFP8) {
          // e4m3 x e4m3: 4 MMAs of K = 32 inside the single 128-byte-wide tile
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_f8_ss(d, dQ + kk * 2u, kb + kk * 2u, id_qk8, kk > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t qo = ((kk >> 2) * 16384u + (kk & 3) * 32u) >> 4;
            const uint32_t ko = ((kk >> 2) * 8192u + (kk & 3) * 32u) >> 4;
            mma_f16_ss(d, dQ + qo, kb + ko, id_qk, kk > 0 ? 1u : 0u);
          }
        }
      };
      auto issue_h = [&](int sl, bool first) {
        const uint64_t pb = dPhi + ((sl * VSLOT) >> 4), vb = dV + ((sl * VSLOT) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16_ss(tmem + T_HK, pb + kk * 128u, vb + kk * 128u, id_h, (first && kk == 0) ? 0u : 1u);
      };
      auto issue_pv = [&](int sl, int b, bool first) {
        const uint32_t pa = tmem + (b ? T_P1 : T_P0);
        if constexpr (kFP8) {
          // P8 (TMEM, 4 keys per column) x V8 (MN-major, one 128-byte atom wide): K = 32 per MMA
          const uint64_t vb = dV8 + ((sl * VSLOT) >> 4);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_f8_ts(tmem + T_O, pa + kk * 8u, vb + kk * 256u, id_pv8, (first && kk == 0) ? 0u : 1u);
        } else {
          const uint64_t vb = dV + ((sl * VSLOT) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ts(tmem + T_O, pa + kk * 8u, vb + kk * 128u, id_pv, (first && kk == 0) ? 0u : 1u);
        }
      };
      // D[col] = A (TMEM, 64 columns of 16-bit pairs) x B (smem MN-major [128 K rows] x 2 chunks of 64 N)
      auto issue_ts128 = [&](uint32_t a_col, uint32_t col, uint32_t idesc, bool first) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ts(tmem + col, tmem + a_col + kk * 8u, dH + kk * 128u, idesc, (first && kk == 0) ? 0u : 1u);
      };

      // Issue order per block i: S_{i+1} (overlaps the softmax of block i), H_i,
      // then PV_i once P_i is in TMEM.  MMA issue is blocking on this hardware
      // (about one instruction per 48-64 cycles), so the issuer waits in
      // suspending barrier tests rather than polling.
      int gk = 0, gv = 0, gs = 0, ti = 0;
      bool ok = true;
      auto issue_s = [&](int b) -> bool {  // S = Q K^T for the next K slot; the slot frees when S is done
        const int sl = gk % kStages;
        if (!mbar_wait(&bars[B_KFULL + sl], (gk / kStages) & 1, abort_flag, a.status)) return false;
        tc_fence_after();
        issue_qk(sl, b);
        mma_commit(&bars[B_SFULL + b]);
        mma_commit(&bars[B_KEMPTY + sl]);
        ++gk;
        return true;
      };
      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++ti) {
        const Tile T = tile_at(a, t, false);
        if (!mbar_wait(&bars[B_QFULL], ti & 1, abort_flag, a.status)) break;
        if (ti > 0 && !mbar_wait(&bars[B_EPIDONE], (ti - 1) & 1, abort_flag, a.status)) break;
        tc_fence_after();
        const int n = T.n_crit;
        if (n > 0 && !issue_s(gs & 1)) break;
        for (int i = 0; ok && i < n; ++i) {
          const int b = (gs + i) & 1, sl = gv % kStages;
          if (i + 1 < n && !issue_s((gs + i + 1) & 1)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&bars[B_VFULL + sl], (gv / kStages) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_h(sl, i == 0);
          if (!mbar_wait(&bars[B_PFULL + b], ((gs + i) >> 1) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(sl, b, i == 0);
          mma_commit(&bars[B_PEMPTY + b]);
          mma_commit(&bars[B_VEMPTY + sl]);
          ++gv;
        }
        for (int i = n; ok && i < T.n_total; ++i) {
          const int sl = gv % kStages;
          if (!mbar_wait(&bars[B_VFULL + sl], (gv / kStages) & 1, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_h(sl, i == 0);
          mma_commit(&bars[B_VEMPTY + sl]);
          ++gv;
        }
        if (!ok) break;
        mma_commit(&bars[B_OFINAL]);
        gs += n;
        if (T.has_lin) {
          if (!mbar_wait(&bars[B_EPI], ti & 1, abort_flag, a.status)) break;
          tc_fence_after();
          issue_ts128(T_PHIQ, T_NUM, idesc_f16(0, 0, 1, 128, 128), true);
          mma_commit(&bars[B_NUM]);
          if (a.wproj != nullptr) {
            if (!mbar_wait(&bars[B_PROJR], ti & 1, abort_flag, a.status)) break;
            tc_fence_after();
            issue_ts128(T_OLHI, T_PROJ, id_bf, true);
            issue_ts128(T_OLLO, T_PROJ, id_bf, false);
            mma_commit(&bars[B_PROJF]);
          }
        }
      }
      // all MMAs must finish before the CTA releases TMEM
      mma_commit(&bars[B_DRAIN]);
      mbar_wait_drain(&bars[B_DRAIN], 0);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 0..7)
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;  // tile row = TMEM lane
    const uint32_t lrow = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t pair_bar = 1 + quarter;  // the two warps that share these rows
    auto RED = [&](int slot, int h) -> float* { return red + (slot * 2 + h) * 128; };
    const bool tail = (a.N & (kBlockKV - 1)) != 0;
    int gs = 0, ti = 0, hc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++ti) {
      const Tile T = tile_at(a, t, false);
      const int tok = T.qb * a.bq + r;
      const bool row_valid = (r < a.bq) && (tok < a.N);
      const float alpha_t = a.alpha ? a.alpha[T.row] : 0.0f;
      const float sigma_t = T.has_lin ? a.sigma[T.bh] : 1.0f;
      const float zt_r = T.has_lin ? a.ztot[static_cast<long long>(T.bh) * kDPad + r] : 0.0f;
      float sl2_q = a.sl2;  // e4m3 branch: times the query block's scale
      if constexpr (kFP8) sl2_q *= a.sq[static_cast<long long>(T.bh) * a.nb128 + (T.qb * a.bq) / 128];
      float m_run = -INFINITY, l_part = 0.0f;
      for (int i = 0; i < T.n_crit; ++i) {
        const int b = (gs + i) & 1;
        ok = ok && warp_wait(&bars[B_SFULL + b], ((gs + i) >> 1) & 1, abort_flag, a.status);
        float s[32];
        if (ok) {
          tc_fence_after();
          tmem_ld32(tmem + lrow + (b ? T_S1 : T_S0) + 32 * half, s);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) s[c] = 0.0f;
        }
        float sc = a.sl2;
        if constexpr (kFP8) {
          const int j = block_at(T, i, a.nkv, nullptr);
          sc = sl2_q * a.sk[static_cast<long long>(T.bh) * a.nb128 + (j >> 1)];  // 128-token key scale block
        }
        if (tail) {
          const int j = block_at(T, i, a.nkv, nullptr);
          if (j == a.nkv - 1) {
            const int nvalid = a.N - j * kBlockKV - 32 * half;
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c >= nvalid) s[c] = -INFINITY;
          }
        }
        float m8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) m8[c] = fmaxf(fmaxf(s[4 * c], s[4 * c + 1]), fmaxf(s[4 * c + 2], s[4 * c + 3]));
        const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        RED(i & 1, half)[r] = mx * sc;
        named_bar_sync(pair_bar, 64);
        const float mt = fmaxf(RED(i & 1, 0)[r], RED(i & 1, 1)[r]);
        // bf16: refresh the max only when it grows by more than 15 (p <= 2^15 fits
        // fp16); e4m3: p * 448 must stay within e4m3, so the exact running max
        const bool need = kFP8 ? (mt > m_run) : (mt > m_run + 15.0f);
        if (__any_sync(0xffffffffu, need)) {
          const float m_new = need ? mt : m_run;
          const float f = need ? ex2_approx(m_run - m_new) : 1.0f;
          if (i > 0) {
            // O holds P V of the previous blocks: wait for the last PV, rescale
            ok = ok && warp_wait(&bars[B_PEMPTY + ((gs + i - 1) & 1)], ((gs + i - 1) >> 1) & 1, abort_flag,
                                 a.status);
            if (ok) {
              tc_fence_after();
#pragma unroll
              for (int cc = 0; cc < 2; ++cc) {
                float o[32];
                tmem_ld32(tmem + lrow + T_O + 64 * half + 32 * cc, o);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) o[c] *= f;
                tmem_st32(tmem + lrow + T_O + 64 * half + 32 * cc, o);
              }
              tmem_wait_st();
            }
          }
          l_part *= f;
          m_run = m_new;
        }
        if (i >= 2) ok = ok && warp_wait(&bars[B_PEMPTY + b], ((gs + i - 2) >> 1) & 1, abort_flag, a.status);
        uint32_t pk[16];
        const float nm = -m_run;
        float l4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if constexpr (kFP8) {
          // p in (0, 1] against the running max; the row sum uses the unquantised p,
          // the PV MMA p * 448 rounded to e4m3 (four keys per TMEM column)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) p[e] = ex2_approx(fmaf(s[4 * c + e], sc, nm));
            l4[c & 3] += (p[0] + p[1]) + (p[2] + p[3]);
            const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(p[0] * 448.0f, p[1] * 448.0f), __NV_SATFINITE,
                                                         __NV_E4M3);
            const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(p[2] * 448.0f, p[3] * 448.0f), __NV_SATFINITE,
                                                         __NV_E4M3);
            pk[c] = lo | (hi << 16);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float p0 = ex2_approx(fmaf(s[2 * c], sc, nm));
            const float p1 = ex2_approx(fmaf(s[2 * c + 1], sc, nm));
            l4[c & 3] += p0 + p1;
            pk[c] = pack_half2(p0, p1);
          }
        }
        l_part += (l4[0] + l4[1]) + (l4[2] + l4[3]);
        if (ok) {
          if constexpr (kFP8)
            tmem_st8(tmem + lrow + (b ? T_P1 : T_P0) + 8 * half, pk);
          else
            tmem_st16(tmem + lrow + (b ? T_P1 : T_P0) + 16 * half, pk);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&bars[B_PFULL + b]);
        }
      }
      gs += T.n_crit;

      // ---------------------------------------------------------- epilogue
      ok = ok && warp_wait(&bars[B_OFINAL], ti & 1, abort_flag, a.status);
      if (ok) tc_fence_after();
      RED(2, half)[r] = l_part;
      named_bar_sync(pair_bar, 64);
      const float l_run = RED(2, 0)[r] + RED(2, 1)[r];
      const float sigma = sigma_t;
      float den = 0.0f;
      if (T.has_lin) {
        // H_i / sigma = H_tot / sigma (fp16 tile from TMA) - H_ex / sigma, row e = r,
        // channels 64*half.., in place in the MN-major H buffer
        ok = ok && warp_wait(&bars[B_HFULL], hc & 1, abort_flag, a.status);
        ++hc;
        const float inv_sigma = 1.0f / sigma;  // exact: sigma is a power of two
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float hk[32];
          if (ok && T.n_total > 0) {
            tmem_ld32(tmem + lrow + T_HK + 64 * half + 32 * cc, hk);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) hk[c] = 0.0f;
          }
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4* hp = reinterpret_cast<uint4*>(sm + OFF_H + half * 16384u + sw128_off(r, 4 * cc + q4));
            const uint4 h8 = *hp;
            const uint32_t hw[4] = {h8.x, h8.y, h8.z, h8.w};
            uint32_t o4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = unpack_half2(hw[e]);
              o4[e] = pack_half2(fmaf(-hk[8 * q4 + 2 * e], inv_sigma, f.x), fmaf(-hk[8 * q4 + 2 * e + 1], inv_sigma, f.y));
            }
            *hp = make_uint4(o4[0], o4[1], o4[2], o4[3]);
          }
        }
        // Z_ex[e] for e = r: this half sums every other listed block's column sums
        {
          const float* zb = a.zblk + static_cast<long long>(T.bh) * a.nkv * kDPad + r;
          float z4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          for (int it = half; it < T.n_total; it += 8) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int i2 = it + 2 * u;
              if (i2 < T.n_total) z4[u] += zb[static_cast<long long>(block_at(T, i2, a.nkv, nullptr)) * kDPad];
            }
          }
          zsh[128 + 128 * half + r] = (z4[0] + z4[1]) + (z4[2] + z4[3]);
        }
        // phi(Q) for row r, channels 64*half .. 64*half+63 (zero past d), fp16 into TMEM
        float x[64];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint4 w;
          if constexpr (kFP8) {  // the smem tile holds e4m3 Q: read the bf16 row (L2-resident)
            w = make_uint4(0, 0, 0, 0);
            if (tok < a.N)
              w = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.qsrc) +
                                                  (static_cast<long long>(T.bh) * a.N + tok) * kDPad + 64 * half + 8 * u);
          } else {
            w = *reinterpret_cast<const uint4*>(sm + OFF_Q + half * 16384u + sw128_off(r, u));
          }
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f2 = unpack_bf162(ww[e]);
            x[8 * u + 2 * e] = f2.x;
            x[8 * u + 2 * e + 1] = f2.y;
          }
        }
        mbar_arrive(&bars[B_QFREE]);  // Q tile no longer read: the next one may load
        const int c0 = 64 * half;
        if (a.phi == SLA_PHI_SOFTMAX) {
          float mx = -INFINITY;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c0 + c < a.d) mx = fmaxf(mx, x[c]);
          RED(0, half)[r] = mx;
          named_bar_sync(pair_bar, 64);
          mx = fmaxf(RED(0, 0)[r], RED(0, 1)[r]);
          float sum = 0.0f;
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            x[c] = (c0 + c < a.d) ? ex2_approx((x[c] - mx) * 1.4426950408889634f) : 0.0f;
            sum += x[c];
          }
          RED(1, half)[r] = sum;
          named_bar_sync(pair_bar, 64);
          const float inv = 1.0f / (RED(1, 0)[r] + RED(1, 1)[r]);
#pragma unroll
          for (int c = 0; c < 64; ++c) x[c] *= inv;
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) x[c] = (c0 + c < a.d) ? elu1(x[c]) : 0.0f;
        }
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          pk[c] = pack_half2(x[2 * c], x[2 * c + 1]);
          const float2 back = unpack_half2(pk[c]);  // the denominator uses the rounded phi(Q)
          x[2 * c] = back.x;
          x[2 * c + 1] = back.y;
        }
        if (ok) {
          tmem_st16(tmem + lrow + T_PHIQ + 32 * half, pk);
          tmem_st16(tmem + lrow + T_PHIQ + 32 * half + 16, pk + 16);
        }
        named_bar_sync(5, kCompute);  // Z_ex halves complete
        if (half == 0) zsh[r] = zt_r - (zsh[128 + r] + zsh[256 + r]);
        named_bar_sync(5, kCompute);  // Z_i complete
        float dp = 0.0f;
#pragma unroll
        for (int c = 0; c < 64; ++c) dp = fmaf(x[c], zsh[c0 + c], dp);
        RED(3, half)[r] = dp;
        named_bar_sync(pair_bar, 64);
        den = RED(3, 0)[r] + RED(3, 1)[r];
        if (ok) {
          tmem_wait_st();
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&bars[B_EPI]);
        }
        ok = ok && warp_wait(&bars[B_NUM], ti & 1, abort_flag, a.status);
        if (ok) tc_fence_after();
      } else {
        mbar_arrive(&bars[B_QFREE]);
      }

      const float inv_l = (T.n_crit > 0 && l_run > 0.0f) ? 1.0f / l_run : 0.0f;
      const float lin_scale = (T.has_lin && den > 0.0f) ? sigma / den : 0.0f;
      const long long obase = (static_cast<long long>(T.bh) * a.N + tok) * a.d;
      uint32_t lin_col = T_NUM;
      float w_s, lin_w;
      if (a.wproj != nullptr) {
        w_s = inv_l;
        lin_w = 1.0f;
        if (T.has_lin) {
          // SLA: O_l -> bf16 hi + lo into TMEM (A operand), W_proj -> smem (MN-major), MMA
          lin_col = T_PROJ;
          float ol[64];
          if (ok) {
            tmem_ld32(tmem + lrow + T_NUM + 64 * half, ol);
            tmem_ld32(tmem + lrow + T_NUM + 64 * half + 32, ol + 32);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int c = 0; c < 64; ++c) ol[c] = 0.0f;
          }
          named_bar_sync(pair_bar, 64);  // both halves have read NUM before it is overwritten
          uint32_t hi[32], lo[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float v0 = ol[2 * c] * lin_scale, v1 = ol[2 * c + 1] * lin_scale;
            hi[c] = pack_bf162(v0, v1);
            const float2 hb = unpack_bf162(hi[c]);
            lo[c] = pack_bf162(v0 - hb.x, v1 - hb.y);
          }
          if (ok) {
            tmem_st16(tmem + lrow + T_OLHI + 32 * half, hi);
            tmem_st16(tmem + lrow + T_OLHI + 32 * half + 16, hi + 16);
            tmem_st16(tmem + lrow + T_OLLO + 32 * half, lo);
            tmem_st16(tmem + lrow + T_OLLO + 32 * half + 16, lo + 16);
          }
          const __nv_bfloat16* wp = static_cast<const __nv_bfloat16*>(a.wproj);
          for (int idx = tid; idx < 128 * 16; idx += kCompute) {
            const int e = idx >> 4, u = idx & 15;
            uint4 w = make_uint4(0, 0, 0, 0);
            if (e < a.d && 8 * u < a.d) w = *reinterpret_cast<const uint4*>(wp + e * a.d + 8 * u);
            *reinterpret_cast<uint4*>(sm + OFF_H + (u >> 3) * 16384u + sw128_off(e, u & 7)) = w;
          }
          if (ok) {
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_PROJR]);
          }
          ok = ok && warp_wait(&bars[B_PROJF], ti & 1, abort_flag, a.status);
          if (ok) tc_fence_after();
        }
      } else {
        w_s = alpha_t * inv_l;
        lin_w = (1.0f - alpha_t) * lin_scale;
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float o[32], nmv[32];
        if (ok && T.n_crit > 0) tmem_ld32(tmem + lrow + T_O + 64 * half + 32 * cc, o);
        if (ok && T.has_lin) tmem_ld32(tmem + lrow + lin_col + 64 * half + 32 * cc, nmv);
        tmem_wait_ld();
        if constexpr (kFP8) {  // O accumulates e4m3 codes: times (absmax_c / 448) / 448 per channel
          const float* va = a.vamax + static_cast<long long>(T.bh) * kDPad + 64 * half + 32 * cc;
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] *= __fdiv_rn(va[c] > 0.0f ? __fdiv_rn(va[c], 448.0f) : __fdiv_rn(1.0f, 448.0f), 448.0f);
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float os = (T.n_crit > 0) ? o[c] * w_s : 0.0f;
          const float olv = T.has_lin ? nmv[c] * lin_w : 0.0f;
          o[c] = os + olv;
        }
        const int ch0 = 64 * half + 32 * cc;
        if (ok && row_valid) {
          if (a.out_bf16) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + obase;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              if (ch0 + 8 * q4 < a.d)
                *reinterpret_cast<uint4*>(dst + ch0 + 8 * q4) =
                    make_uint4(pack_bf162(o[8 * q4], o[8 * q4 + 1]), pack_bf162(o[8 * q4 + 2], o[8 * q4 + 3]),
                               pack_bf162(o[8 * q4 + 4], o[8 * q4 + 5]), pack_bf162(o[8 * q4 + 6], o[8 * q4 + 7]));
          } else {
            float* dst = static_cast<float*>(a.out) + obase;
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              if (ch0 + 4 * q4 < a.d)
                *reinterpret_cast<float4*>(dst + ch0 + 4 * q4) =
                    make_float4(o[4 * q4], o[4 * q4 + 1], o[4 * q4 + 2], o[4 * q4 + 3]);
          }
        }
      }
      if (ok) {
        tc_fence_before();
        mbar_arrive(&bars[B_EPIDONE]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

template <bool kFP8>
static cudaError_t launch_sparse_t(const SparseArgs& a, const CUtensorMap& mq, const CUtensorMap& mk,
                                   const CUtensorMap& mp, const CUtensorMap& mv, const CUtensorMap& mh,
                                   const CUtensorMap& mv8, cudaStream_t st) {
  constexpr uint32_t smem = Lay<kFP8>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(sparse_fwd_kernel<kFP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = kNumSMs;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long ntiles = static_cast<long long>(a.BH) * a.nq;
  const unsigned grid = static_cast<unsigned>(ntiles < sms ? ntiles : sms);
  sparse_fwd_kernel<kFP8><<<grid, kThreads, smem, st>>>(mq, mk, mp, mv, mh, mv8, a);
  return cudaGetLastError();
}

cudaError_t launch_sparse(const SparseArgs& a, const void* q_bf16_128, const void* k_bf16_128,
                          const void* phik16, const void* v16, const void* hs16, const void* q8, const void* k8,
                          const void* v8, cudaStream_t st) {
  CUtensorMap mq, mk, mp, mv, mh, mv8;
  cudaError_t e;
  if ((e = encode_map(&mp, phik16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.N, a.BH, 64)) != cudaSuccess) return e;
  if ((e = encode_map(&mv, v16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.N, a.BH, 64)) != cudaSuccess) return e;
  if ((e = encode_map(&mh, hs16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, kDPad, a.BH, 128)) != cudaSuccess) return e;
  if (a.fp8) {
    if ((e = encode_map8(&mq, q8, a.N, a.BH, 128)) != cudaSuccess) return e;
    if ((e = encode_map8(&mk, k8, a.N, a.BH, 64)) != cudaSuccess) return e;
    if ((e = encode_map8(&mv8, v8, a.N, a.BH, 64)) != cudaSuccess) return e;
    return launch_sparse_t<true>(a, mq, mk, mp, mv, mh, mv8, st);
  }
  if ((e = encode_map(&mq, q_bf16_128, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.N, a.BH, 128)) != cudaSuccess) return e;
  if ((e = encode_map(&mk, k_bf16_128, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.N, a.BH, 64)) != cudaSuccess) return e;
  return launch_sparse_t<false>(a, mq, mk, mp, mv, mh, mv, st);
}

}  // namespace sla
