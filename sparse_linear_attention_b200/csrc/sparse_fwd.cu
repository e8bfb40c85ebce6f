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
// (b, h, query block) in head-major order.  The listed key blocks of a tile
// are taken two at a time ("steps" of 128 keys): one N = 128 tensor-core
// product per step for S, and one max exchange per 128 keys.  352 threads:
//   warp 8      TMA producer, running ahead across tiles: per step the two
//               key tiles side by side in one 128-row slot of a 2-slot ring
//               (freed once S has read it); per step the phi(K), V tiles
//               (fp16) of its two blocks in one entry of a 2-entry ring (freed
//               after PV and H); per tile the Q tile (as soon as the previous
//               tile's S products are done) and, in the ring entry after its
//               blocks, the fp16 H_tot / sigma tile of its head.
//   warps 9, 10 tcgen05 issuers (one thread each), fp32 accumulators in TMEM.
//               Warp 9:   S = Q [K_a | K_b]^T  (bf16 operands in smem) and
//                         O += [P_a | P_b] [V_a ; V_b] (fp16 P from TMEM), in
//                         the order S_{i+1}, PV_i so S runs ahead of the softmax.
//               Warp 10:  H_ex += phi(K_j)^T V_j (fp16), and per tile
//                         phi(Q) H_i / sigma (phi(Q) in TMEM), for SLA also
//                         O_l W_proj (bf16 hi + lo split).
//               Two issuers keep the tensor pipe fed with H work while warp 9
//               waits for P.
//   warps 0..7  softmax and epilogue: warp w owns query rows 32(w%4)..+31
//               (its TMEM lane quarter) and key / channel half w/4 (one of
//               the two key blocks of a step), so two warps share each row.
//               Online softmax in log2 units; the running max is refreshed
//               only when a step's max exceeds it by more than 15 (exact: the
//               stale max scales numerator and denominator alike, and
//               p <= 2^15 still fits fp16).  P is rounded to fp16 and written
//               over the step's S columns in TMEM for the PV product.
//               phi(Q) of a tile is formed (packed in registers) during the
//               previous tile's epilogue, while phi(Q) H_i runs, so the Q tile
//               in smem is replaced early.  The epilogue does the work that
//               needs no product (row sums, Z_i, the denominator) and H_i
//               (once warp 10's products are done) before it waits for the
//               last PV; the output store's smem read is waited for only
//               after the next tile's first step.
// TMEM (512 columns): S0 | S1 (128 each, P over part of them) | O (128) |
// H_ex (128, then phi(Q) H_i or the SLA projection in the epilogue).
// The linear branch uses H_i = H_tot - sum over the listed blocks of
// phi(K_j)^T V_j (H_tot from sla_prepare) and Z_i = Z_tot - the listed
// blocks' column sums of phi(K), summed during the steps.  H_i enters the
// product as fp16 scaled by an exact power of two sigma >= max_e Z_tot[e],
// which bounds |H_i / sigma| by max|V|.
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

constexpr int kThreads = 352;  // 8 softmax warps, producer, two MMA issuers
constexpr int kCompute = 256;
constexpr int kKSlots = 2;  // key-pair slots
constexpr int kVSlots = 2;  // value entries: the phi(K) | V tiles of a step's two blocks, or the H tile

// Shared-memory layout (the dynamic shared window is 1024-byte aligned).
//   bf16 branch: Q tile 2 x [128 rows][128 B]; key-pair slot
//     [chunk 0: A rows | B rows][chunk 1: A rows | B rows] (128 rows per
//     chunk); V slot = phi(K) | V (fp16, each 2 x [64 rows][128 B]).
//   e4m3 branch: Q8 [128 rows][128 B]; key-pair slot [A rows | B rows] x
//     128 B; V slot = phi(K) | V (fp16) | V8 [64 rows][128 B].
// then barriers, flags, the row-pair exchange buffer and Z_i.
template <bool kFP8>
struct Lay {
  static constexpr uint32_t QBYTES = kFP8 ? 16384 : 32768;
  static constexpr uint32_t KBLK = kFP8 ? 8192 : 16384;  // bytes of one key block
  static constexpr uint32_t KSLOT = 2 * KBLK;
  static constexpr uint32_t VBLK = kFP8 ? 40960 : 32768;  // one key block's phi(K) | V (| V8)
  static constexpr uint32_t VSLOT = 2 * VBLK;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = QBYTES;
  static constexpr uint32_t OFF_V = OFF_K + kKSlots * KSLOT;
  static constexpr uint32_t OFF_BAR = OFF_V + kVSlots * VSLOT;
  static constexpr uint32_t OFF_MISC = OFF_BAR + 256;  // tmem base, abort flag
  static constexpr uint32_t OFF_RED = OFF_MISC + 64;   // [2 slots][2 halves][128 rows] floats
  static constexpr uint32_t OFF_Z = OFF_RED + 2048;    // Z_i [128] floats
  static constexpr uint32_t SMEM_BYTES = OFF_Z + 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && VBLK % 1024 == 0, "1 KB aligned tiles");
};

// TMEM columns (512 allocated; one CTA per SM)
constexpr uint32_t T_S0 = 0;     // S buffer b at T_S0 + 128 b; each key block's P over the first 32 (bf16) /
                                 // 16 (e4m3) columns of its 64
constexpr uint32_t T_O = 256;    // O accumulator
constexpr uint32_t T_HK = 384;   // H_ex accumulator; epilogue: phi(Q) H_i, then O_l W_proj
constexpr uint32_t TMEM_COLS = 512;

enum {
  B_QFULL = 0,
  B_QFREE = 1,    // the 256 softmax threads have read the Q tile + MMA commit after its last S
  B_KFULL = 2,    // +slot; a key-pair slot is free again once S of its step is done (B_SFULL)
  B_VFULL = 4,    // +slot
  B_VEMPTY = 6,   // +slot
  B_SFULL = 8,    // +buffer (= key-pair slot)
  B_PFULL = 10,   // +buffer
  B_PEMPTY = 12,  // +buffer
  B_OFINAL = 14,  // warp 9's products of the tile (its last PV) are done
  B_EPI = 15,
  B_NUM = 16,
  B_EPIDONE = 17,
  B_PROJR = 18,
  B_PROJF = 19,
  B_DRAIN = 20,   // +issuer (2)
  B_HFIN = 22,    // warp 10's products of the tile (H_ex) are done
  NBAR = 23
};
static_assert(NBAR * 8 <= 256, "barrier area");

struct Tile {
  int bh, qb;
  long long row;
  int n_crit, n_negl, n_total, nsteps, nnegl_e;  // nnegl_e: value entries of negligible blocks (two per entry)
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
  T.nsteps = (T.n_crit + 1) >> 1;
  T.nnegl_e = (T.n_negl + 1) >> 1;
  T.crit = a.crit_idx + T.row * a.list_stride;
  T.negl = a.negl_idx ? a.negl_idx + T.row * a.list_stride : T.crit;
  T.has_lin = (a.nkv - T.n_total) > 0;
  return T;
}

// Key block at list position it (critical blocks first, then negligible ones);
// an index outside [0, n_kv) is reported and replaced by 0.
__device__ __forceinline__ int block_at(const Tile& T, int it, int nkv, int* status) {
  int j = it < T.n_crit ? T.crit[it] : T.negl[it - T.n_crit];
  if (j < 0 || j >= nkv) {
    if (status) report_error(status, SLA_ERR_DEVICE_INDEX);
    j = 0;
  }
  return j;
}

// Warp-uniform bounded wait: every lane polls, the warp agrees on the verdict.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* status, uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status, limit_ns);
  return __all_sync(0xffffffffu, ok) != 0;
}

// kLow: 0 = bf16 sparse branch; 1 = e4m3 Q, K', P, V; 2 = INT8 Q, K' (S as an
// exact integer product, kind::i8) with e4m3 P, V.  kStats: the backward's
// per-row statistics epilogue (SparseArgs::bwd_rows; bf16 branch only).
template <int kLow, bool kStats>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmPhi, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmV8,
                      const __grid_constant__ CUtensorMap tmO, const SparseArgs a) {
  constexpr bool kFP8 = kLow != 0;  // the low-bit layout (8-bit Q, K', V)
  constexpr bool kI8 = kLow == 2;
  using L = Lay<kFP8>;
  constexpr uint32_t OFF_Q = L::OFF_Q, OFF_K = L::OFF_K, OFF_V = L::OFF_V;
  constexpr uint32_t OFF_BAR = L::OFF_BAR, OFF_MISC = L::OFF_MISC, OFF_RED = L::OFF_RED, OFF_Z = L::OFF_Z;
  constexpr uint32_t KBLK = L::KBLK, KSLOT = L::KSLOT, VBLK = L::VBLK, VSLOT = L::VSLOT;
  extern __shared__ __align__(1024) uint8_t sm[];
  // The swizzled tiles need a 1024-byte aligned window; the runtime gives one
  // when the kernel has no static shared memory.  Check rather than assume.
  if ((smem_u32(sm) & 1023u) != 0) {
    if (threadIdx.x == 0) report_error(a.status, SLA_ERR_UNSUPPORTED);
    return;
  }
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
    mbar_init(&bars[B_QFREE], kCompute + 1);
    for (int s = 0; s < kKSlots; ++s) mbar_init(&bars[B_KFULL + s], 1);
    for (int s = 0; s < kVSlots; ++s) {
      mbar_init(&bars[B_VFULL + s], 1);
      mbar_init(&bars[B_VEMPTY + s], 2);  // released by both issuers
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[B_SFULL + b], 1);
      mbar_init(&bars[B_PFULL + b], kCompute);
      mbar_init(&bars[B_PEMPTY + b], 1);
    }
    mbar_init(&bars[B_OFINAL], 1);
    mbar_init(&bars[B_HFIN], 1);
    mbar_init(&bars[B_EPI], kCompute);
    mbar_init(&bars[B_NUM], 1);
    mbar_init(&bars[B_EPIDONE], kCompute);
    mbar_init(&bars[B_PROJR], kCompute);
    mbar_init(&bars[B_PROJF], 1);
    mbar_init(&bars[B_DRAIN], 1);
    mbar_init(&bars[B_DRAIN + 1], 1);
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
      int gk = 0, gv = 0, q_issued = 0;
      bool ok = true;
      // the key tiles of step s (list positions 2s, 2s+1) into the next pair slot
      auto load_k = [&](const Tile& T, int s) -> bool {
        const int sl = gk % kKSlots;
        if (gk >= kKSlots && !mbar_wait(&bars[B_SFULL + sl], ((gk / kKSlots) - 1) & 1, abort_flag, a.status, a.wait_ns))
          return false;  // S of the step two back has read this slot
        const bool two = 2 * s + 1 < T.n_crit;
        const int ra = block_at(T, 2 * s, a.nkv, a.status) * kBlockKV;
        const int rb = two ? block_at(T, 2 * s + 1, a.nkv, a.status) * kBlockKV : 0;
        uint64_t* fb = &bars[B_KFULL + sl];
        uint8_t* kb = sm + OFF_K + sl * KSLOT;
        mbar_arrive_expect_tx(fb, two ? 2 * KBLK : KBLK);
        if constexpr (kFP8) {
          tma_load_3d(kb, &tmK, fb, 0, ra, T.bh);
          if (two) tma_load_3d(kb + 8192, &tmK, fb, 0, rb, T.bh);
        } else {
          tma_load_3d(kb, &tmK, fb, 0, ra, T.bh);
          tma_load_3d(kb + 16384, &tmK, fb, 64, ra, T.bh);
          if (two) {
            tma_load_3d(kb + 8192, &tmK, fb, 0, rb, T.bh);
            tma_load_3d(kb + 16384 + 8192, &tmK, fb, 64, rb, T.bh);
          }
        }
        ++gk;
        return true;
      };
      auto v_slot = [&](uint64_t*& fb) -> uint8_t* {
        const int sl = gv % kVSlots;
        if (gv >= kVSlots && !mbar_wait(&bars[B_VEMPTY + sl], ((gv / kVSlots) - 1) & 1, abort_flag, a.status, a.wait_ns))
          return nullptr;
        fb = &bars[B_VFULL + sl];
        ++gv;
        return sm + OFF_V + sl * VSLOT;
      };
      // phi(K), V (and V8) tiles of the blocks at list positions p0 and p0 + 1 (if below p_end)
      auto load_pair = [&](const Tile& T, int p0, int p_end) -> bool {
        uint64_t* fb = nullptr;
        uint8_t* vb = v_slot(fb);
        if (vb == nullptr) return false;
        const int nb = p0 + 1 < p_end ? 2 : 1;
        mbar_arrive_expect_tx(fb, nb * VBLK);
        for (int b = 0; b < nb; ++b) {
          const int krow = block_at(T, p0 + b, a.nkv, a.status) * kBlockKV;
          uint8_t* bb = vb + b * VBLK;
          tma_load_3d(bb, &tmPhi, fb, 0, krow, T.bh);
          tma_load_3d(bb + 8192, &tmPhi, fb, 64, krow, T.bh);
          tma_load_3d(bb + 16384, &tmV, fb, 0, krow, T.bh);
          tma_load_3d(bb + 16384 + 8192, &tmV, fb, 64, krow, T.bh);
          if constexpr (kFP8) tma_load_3d(bb + 32768, &tmV8, fb, 0, krow, T.bh);
        }
        return true;
      };
      auto load_h = [&](const Tile& T) -> bool {
        uint64_t* fb = nullptr;
        uint8_t* hb = v_slot(fb);
        if (hb == nullptr) return false;
        mbar_arrive_expect_tx(fb, 32768);
        tma_load_3d(hb, &tmH, fb, 0, 0, T.bh);
        tma_load_3d(hb + 16384, &tmH, fb, 64, 0, T.bh);
        return true;
      };
      int ti = 0;
      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++ti) {
        const Tile T = tile_at(a, t, true);
        if (ti > 0 && !mbar_wait(&bars[B_QFREE], (ti - 1) & 1, abort_flag, a.status, a.wait_ns)) break;
        mbar_arrive_expect_tx(&bars[B_QFULL], L::QBYTES);
        tma_load_3d(sm + OFF_Q, &tmQ, &bars[B_QFULL], 0, T.qb * a.bq, T.bh);
        if constexpr (!kFP8) tma_load_3d(sm + OFF_Q + 16384, &tmQ, &bars[B_QFULL], 64, T.qb * a.bq, T.bh);
        q_issued = ti + 1;
        // key pairs run one step ahead of the value blocks
        if (T.nsteps > 0) ok = load_k(T, 0);
        if (ok && T.nsteps > 1) ok = load_k(T, 1);
        for (int s = 0; ok && s < T.nsteps; ++s) {
          ok = load_pair(T, 2 * s, T.n_crit);
          if (ok && s + 2 < T.nsteps) ok = load_k(T, s + 2);
        }
        for (int it = T.n_crit; ok && it < T.n_total; it += 2) ok = load_pair(T, it, T.n_total);
        if (ok && T.has_lin) ok = load_h(T);
      }
      // every issued copy must land before the CTA may exit
      if (q_issued > 0) mbar_wait_drain(&bars[B_QFULL], (q_issued - 1) & 1);
      for (int g = gk > kKSlots ? gk - kKSlots : 0; g < gk; ++g)
        mbar_wait_drain(&bars[B_KFULL + g % kKSlots], (g / kKSlots) & 1);
      for (int g = gv > kVSlots ? gv - kVSlots : 0; g < gv; ++g)
        mbar_wait_drain(&bars[B_VFULL + g % kVSlots], (g / kVSlots) & 1);
    }
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 9 issues S and PV (the chain through the softmax), warp 10 the
    // phi(K)^T V products and the epilogue products, so the tensor pipe gets
    // H work while warp 9 waits for P.  Both walk the V ring and release each
    // entry once its data has landed and their products on it are done.
    if (lane == 0) {
      const bool sp = warp == 9;
      const uint32_t id_qk = idesc_f16(1, 0, 0, 128, 128);  // Q (K-major) x [K_a|K_b] (K-major), bf16
      const uint32_t id_qk1 = idesc_f16(1, 0, 0, 128, 64);  // one key block
      const uint32_t id_h = idesc_f16(0, 1, 1, 128, 128);   // phi(K)^T (MN-major) x V (MN-major), f16
      const uint32_t id_pv = idesc_f16(0, 0, 1, 128, 128);  // TMEM A (f16) x MN-major B
      const uint32_t id_bf = idesc_f16(1, 0, 1, 128, 128);  // TMEM A (bf16) x MN-major B
      const uint32_t id_qk8 = idesc_f8(0, 0, 128, 128);     // Q8 x [K8_a|K8_b], e4m3
      const uint32_t id_qk81 = idesc_f8(0, 0, 128, 64);
      const uint32_t id_qki8 = idesc_i8(0, 0, 128, 128);    // Q8 x [K8_a|K8_b], INT8, s32 accumulate
      const uint32_t id_qki81 = idesc_i8(0, 0, 128, 64);
      const uint32_t id_pv8 = idesc_f8(0, 1, 128, 128);     // P8 (TMEM) x V8 (MN-major), e4m3
      // Descriptors built once; a byte offset d inside the window adds d >> 4 to
      // the start-address field (addresses stay below 2^18, so it cannot carry).
      const uint64_t dQ = sdesc_sw128(smem_u32(sm + OFF_Q), 16, 1024);
      const uint64_t dK = sdesc_sw128(smem_u32(sm + OFF_K), 16, 1024);
      const uint64_t dPhi = sdesc_sw128(smem_u32(sm + OFF_V), 8192, 1024);
      const uint64_t dV = sdesc_sw128(smem_u32(sm + OFF_V) + 16384, 8192, 1024);
      const uint64_t dV8 = sdesc_sw128(smem_u32(sm + OFF_V) + 32768, 16, 1024);  // MN-major, N fits one atom
      const uint64_t dH = sdesc_sw128(smem_u32(sm + OFF_V), 16384, 1024);       // H tile / W_proj in a V slot
      int gk = 0, gv = 0, gs = 0, ti = 0;
      bool ok = true;
      // The first barrier test after products that read both operands from
      // smem stalls until their reads drain (~300 cycles); after products
      // with A in TMEM it costs little.  So warp 9 waits for all of a step's
      // data right after the previous PV.
      auto wait_k = [&]() -> bool {  // the next key pair has landed (TMA data: no tcgen05 fence needed)
        const int sl = gk % kKSlots;
        return mbar_wait(&bars[B_KFULL + sl], (gk / kKSlots) & 1, abort_flag, a.status, a.wait_ns);
      };
      // S for step s of T into buffer g & 1 (key pair already waited for); frees the slot when done
      auto issue_s = [&](const Tile& T, int s, int g, bool last_s) {
        const int sl = gk % kKSlots;
        const bool two = 2 * s + 1 < T.n_crit;
        const uint64_t kb = dK + ((sl * KSLOT) >> 4);
        const uint32_t d = tmem + T_S0 + (g & 1) * 128;
        if constexpr (kFP8) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            if constexpr (kI8)
              mma_i8_ss(d, dQ + kk * 2u, kb + kk * 2u, two ? id_qki8 : id_qki81, kk > 0 ? 1u : 0u);
            else
              mma_f8_ss(d, dQ + kk * 2u, kb + kk * 2u, two ? id_qk8 : id_qk81, kk > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t o = ((kk >> 2) * 16384u + (kk & 3) * 32u) >> 4;  // same offsets in Q and the pair slot
            mma_f16_ss(d, dQ + o, kb + o, two ? id_qk : id_qk1, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(&bars[B_SFULL + (g & 1)]);  // also frees key-pair slot g & 1 (== sl)
        if (last_s) mma_commit(&bars[B_QFREE]);
        ++gk;
      };
      auto take_v = [&]() -> int {  // next V-ring entry, once it has landed
        const int sl = gv % kVSlots;
        if (!mbar_wait(&bars[B_VFULL + sl], (gv / kVSlots) & 1, abort_flag, a.status, a.wait_ns)) return -1;
        ++gv;
        return sl;
      };
      auto issue_h = [&](int sl, int blk, bool first) {
        const uint32_t off = (sl * VSLOT + blk * VBLK) >> 4;
        const uint64_t pb = dPhi + off, vb = dV + off;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16_ss(tmem + T_HK, pb + kk * 128u, vb + kk * 128u, id_h, (first && kk == 0) ? 0u : 1u);
      };
      // O (+)= P V for one key block: P columns from pcol, V of block blk of entry sl
      auto issue_pv = [&](int sl, int blk, uint32_t pcol, bool first) {
        const uint32_t off = (sl * VSLOT + blk * VBLK) >> 4;
        if constexpr (kFP8) {
          // P8 (TMEM, 4 keys per column) x V8 (MN-major, one 128-byte atom wide): K = 32 per MMA
          const uint64_t vb = dV8 + off;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_f8_ts(tmem + T_O, tmem + pcol + kk * 8u, vb + kk * 256u, id_pv8, (first && kk == 0) ? 0u : 1u);
        } else {
          const uint64_t vb = dV + off;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ts(tmem + T_O, tmem + pcol + kk * 8u, vb + kk * 128u, id_pv, (first && kk == 0) ? 0u : 1u);
        }
      };
      // D[col] = A (TMEM, 64 columns of 16-bit pairs) x B (smem MN-major [128 K rows] x 2 chunks of 64 N)
      auto issue_ts128 = [&](uint32_t a_col, uint32_t col, uint64_t b, uint32_t idesc, bool first) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ts(tmem + col, tmem + a_col + kk * 8u, b + kk * 128u, idesc, (first && kk == 0) ? 0u : 1u);
      };
      bool pend = false;  // the previous tile's epilogue is outstanding
      int pend_ti = 0;
      auto wait_epidone = [&]() -> bool {
        pend = false;
        if (!mbar_wait(&bars[B_EPIDONE], pend_ti & 1, abort_flag, a.status, a.wait_ns)) return false;
        tc_fence_after();
        return true;
      };

      for (int t = blockIdx.x; ok && t < ntiles; t += gridDim.x, ++ti) {
        const Tile T = tile_at(a, t, false);
        if (sp) {
          // ---------------------------------------------- warp 9: S, PV
          if (!mbar_wait(&bars[B_QFULL], ti & 1, abort_flag, a.status, a.wait_ns)) break;
          tc_fence_after();
          const int ns = T.nsteps;
          if (ns > 0) {
            if (!wait_k()) break;
            issue_s(T, 0, gs, ns == 1);
          }
          if (ns == 0) mma_commit(&bars[B_QFREE]);
          if (pend && !wait_epidone()) break;  // O is free again
          for (int i = 0; ok && i < ns; ++i) {
            const int g = gs + i, b = g & 1;
            const bool two = 2 * i + 1 < T.n_crit;
            if (i + 1 < ns) {  // right after the previous PV: a cheap place to wait
              if (!wait_k()) {
                ok = false;
                break;
              }
              issue_s(T, i + 1, g + 1, i + 1 == ns - 1);
            }
            if (!mbar_wait(&bars[B_PFULL + b], (g >> 1) & 1, abort_flag, a.status, a.wait_ns)) {
              ok = false;
              break;
            }
            const int ve = take_v();  // (this step's blocks: long landed)
            if (ve < 0) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t pcol = T_S0 + b * 128;
            issue_pv(ve, 0, pcol, i == 0);
            if (two) issue_pv(ve, 1, pcol + 64u, false);  // block B's P over the first columns of its S half
            mma_commit(&bars[B_PEMPTY + b]);
            mma_commit(&bars[B_VEMPTY + ve]);
          }
          // the tile's other value entries (negligible blocks, H tile) are warp 10's
          for (int it = 0; ok && it < T.nnegl_e + (T.has_lin ? 1 : 0); ++it) {
            const int sl = take_v();
            if (sl < 0) {
              ok = false;
              break;
            }
            mma_commit(&bars[B_VEMPTY + sl]);
          }
          if (!ok) break;
          mma_commit(&bars[B_OFINAL]);
          gs += ns;
        } else {
          // ---------------------------------------------- warp 10: H, epilogue products
          if (pend && !wait_epidone()) break;  // H_ex, phi(Q) H_i of the previous tile have been read
          for (int e = 0; ok && e < T.nsteps + T.nnegl_e; ++e) {
            const int sl = take_v();
            if (sl < 0) {
              ok = false;
              break;
            }
            const int p0 = e < T.nsteps ? 2 * e : T.n_crit + 2 * (e - T.nsteps);
            const int p_end = e < T.nsteps ? T.n_crit : T.n_total;
            issue_h(sl, 0, e == 0);  // (TMA data: no tcgen05 fence needed)
            if (p0 + 1 < p_end) issue_h(sl, 1, false);
            mma_commit(&bars[B_VEMPTY + sl]);
          }
          if (!ok) break;
          mma_commit(&bars[B_HFIN]);
          // epilogue: phi(Q) (TMEM, the tile's last S buffer) x H_i / sigma (smem, the H tile's slot)
          if (!mbar_wait(&bars[B_EPI], ti & 1, abort_flag, a.status, a.wait_ns)) break;
          tc_fence_after();
          const uint32_t ecol = T_S0 + ((gs + T.nsteps - 1) & 1) * 128;
          gs += T.nsteps;
          int hs = 0;
          if (T.has_lin) {
            hs = take_v();
            if (hs < 0) break;
            issue_ts128(ecol, T_HK, dH + ((hs * VSLOT) >> 4), id_pv, true);
          }
          mma_commit(&bars[B_NUM]);
          if (a.wproj != nullptr) {
            if (!mbar_wait(&bars[B_PROJR], ti & 1, abort_flag, a.status, a.wait_ns)) break;
            tc_fence_after();
            if (T.has_lin) {
              const uint64_t hb = dH + ((hs * VSLOT) >> 4);
              issue_ts128(ecol, T_HK, hb, id_bf, true);        // O_l hi x W_proj
              issue_ts128(ecol + 64, T_HK, hb, id_bf, false);  // O_l lo x W_proj
            }
            mma_commit(&bars[B_PROJF]);
          }
          if (T.has_lin && !a.tma_out) mma_commit(&bars[B_VEMPTY + hs]);  // else released after the output store
        }
        pend = true;
        pend_ti = ti;
      }
      // all MMAs must finish before the CTA releases TMEM
      mma_commit(&bars[B_DRAIN + (sp ? 0 : 1)]);
      mbar_wait_drain(&bars[B_DRAIN + (sp ? 0 : 1)], 0);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 0..7)
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;  // tile row = TMEM lane
    const uint32_t lrow = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t pair_bar = 1 + quarter;  // the two warps that share these rows
    const bool tail = (a.N & (kBlockKV - 1)) != 0;
    int gs = 0, ti = 0, gv = 0, xc = 0;
    bool ok = true;
    // value exchange with the other warp of the row pair (two alternating slots)
    auto xchg = [&](float v) -> float {
      float* base = red + (xc & 1) * 256;
      base[half * 128 + r] = v;
      named_bar_sync(pair_bar, 64);
      const float o = base[(1 - half) * 128 + r];
      ++xc;
      return o;
    };
    // Lane l holds the block of this half at step 32 c + l of the current
    // chunk c (one coalesced load per 32 steps); steps read it by shuffle.
    auto list_chunk = [&](const Tile& T, int c) -> int {
      const int p = 2 * (32 * c + lane) + half;
      if (p >= T.n_crit) return -1;
      const int j = T.crit[p];
      return (j < 0 || j >= a.nkv) ? 0 : j;
    };
    // phi(Q) of tile Tq for row r, channels 64*half .. 64*half+63 (zero past d),
    // packed fp16 into phq.  Formed as soon as the tile's Q lands (for every tile
    // after the first, while the previous tile's epilogue products run), so the
    // Q tile can be replaced early.
    uint32_t phq[32];
    auto form_phi_q = [&](const Tile& Tq, int tiq) {
      ok = ok && warp_wait(&bars[B_QFULL], tiq & 1, abort_flag, a.status, a.wait_ns);
      const int tokq = Tq.qb * a.bq + r;
      {
        uint4 qw[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          qw[u] = make_uint4(0, 0, 0, 0);
          if (Tq.has_lin) {
            if constexpr (kFP8) {  // the smem tile holds e4m3 Q: read the bf16 row
              if (tokq < a.N)
                qw[u] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.qsrc) +
                                                        (static_cast<long long>(Tq.bh) * a.N + tokq) * kDPad + 64 * half + 8 * u);
            } else {
              qw[u] = *reinterpret_cast<const uint4*>(sm + OFF_Q + half * 16384u + sw128_off(r, u));
            }
          }
        }
        mbar_arrive(&bars[B_QFREE]);  // this thread no longer reads the Q tile
        const int c0 = 64 * half;
        if (a.phi == SLA_PHI_SOFTMAX) {
          float mx = -INFINITY;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t ww[4] = {qw[u].x, qw[u].y, qw[u].z, qw[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f2 = unpack_bf162(ww[e]);
              if (c0 + 8 * u + 2 * e < a.d) mx = fmaxf(mx, f2.x);
              if (c0 + 8 * u + 2 * e + 1 < a.d) mx = fmaxf(mx, f2.y);
            }
          }
          mx = fmaxf(mx, xchg(mx));
          float sum = 0.0f;
          float y[64];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t ww[4] = {qw[u].x, qw[u].y, qw[u].z, qw[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f2 = unpack_bf162(ww[e]);
              const int c = 8 * u + 2 * e;
              const float e0 = ex2_approx((f2.x - mx) * 1.4426950408889634f);  // evaluated, then selected
              const float e1 = ex2_approx((f2.y - mx) * 1.4426950408889634f);
              y[c] = (c0 + c < a.d) ? e0 : 0.0f;
              y[c + 1] = (c0 + c + 1 < a.d) ? e1 : 0.0f;
              sum += y[c] + y[c + 1];
            }
          }
          const float inv = 1.0f / (sum + xchg(sum));
#pragma unroll
          for (int c = 0; c < 32; ++c) phq[c] = pack_half2(y[2 * c] * inv, y[2 * c + 1] * inv);
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t ww[4] = {qw[u].x, qw[u].y, qw[u].z, qw[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f2 = unpack_bf162(ww[e]);
              const int c = 8 * u + 2 * e;
              const float e0 = elu1(f2.x), e1 = elu1(f2.y);  // evaluated, then selected: no branch
              phq[4 * u + e] = pack_half2((c0 + c < a.d) ? e0 : 0.0f, (c0 + c + 1 < a.d) ? e1 : 0.0f);
            }
          }
        }
      }
    };
    if (blockIdx.x < ntiles) form_phi_q(tile_at(a, blockIdx.x, false), 0);
    // The previous tile's output store may still read its smem slot: thread 0
    // waits for that read and frees the slot after the next tile's first step.
    bool pend_store = false;
    int pend_hsl = 0;
    auto release_store = [&]() {
      if (pend_store) {
        if (tid == 0) {
          bulk_wait_read_all();
          mbar_arrive(&bars[B_VEMPTY + pend_hsl]);
        }
        pend_store = false;
      }
    };
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++ti) {
      const Tile T = tile_at(a, t, false);
      const int tok = T.qb * a.bq + r;
      const bool row_valid = (r < a.bq) && (tok < a.N);
      float sl2_q = a.sl2;  // e4m3 branch: times the query block's scale
      if constexpr (kFP8) sl2_q *= a.sq[static_cast<long long>(T.bh) * a.nb128 + (T.qb * a.bq) / 128];
      int jl = list_chunk(T, 0);
      const float alpha_t = a.alpha ? a.alpha[T.row] : 0.0f;
      const float sigma = T.has_lin ? a.sigma[T.bh] : 1.0f;
      const float zt_r = T.has_lin ? a.ztot[static_cast<long long>(T.bh) * kDPad + r] : 0.0f;

      // ---------------------------------------------------------- steps of two key blocks
      float m_run = -INFINITY, l_part = 0.0f, zex = 0.0f;
      const float* zb = a.zblk + static_cast<long long>(T.bh) * a.nkv * kDPad + r;
      for (int i = 0; i < T.nsteps; ++i) {
        const int g = gs + i, b = g & 1;
        if (i > 0 && (i & 31) == 0) jl = list_chunk(T, i >> 5);
        const int j_cur = __shfl_sync(0xffffffffu, jl, i & 31);
        const float zv = (T.has_lin && j_cur >= 0) ? zb[static_cast<long long>(j_cur) * kDPad] : 0.0f;
        ok = ok && warp_wait(&bars[B_SFULL + b], (g >> 1) & 1, abort_flag, a.status, a.wait_ns);
        const bool live = ok && j_cur >= 0;  // this half has a key block in this step
        const uint32_t scol = tmem + lrow + T_S0 + b * 128 + 64 * half;  // this half's 64 S columns
        const int nvalid = (tail && j_cur == a.nkv - 1) ? a.N - j_cur * kBlockKV : kBlockKV;
        float sc = a.sl2;
        if constexpr (kFP8) {
          if (j_cur >= 0) sc = sl2_q * a.sk[static_cast<long long>(T.bh) * a.nb128 + (j_cur >> 1)];  // 128-token key block
        }
        // pass 1: the block's row max (keys past N masked)
        float mx = -INFINITY;
        if (live) {
          tc_fence_after();
          float s[64];
          tmem_ld32(scol, s);
          tmem_ld32(scol + 32, s + 32);
          tmem_wait_ld();
          if constexpr (kI8) {  // s32 accumulators: exact below 2^24, so the conversion is exact
#pragma unroll
            for (int c = 0; c < 64; ++c) s[c] = static_cast<float>(__float_as_int(s[c]));
          }
          if (nvalid < kBlockKV) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c >= nvalid) s[c] = -INFINITY;
          }
          float m8[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            m8[c] = fmaxf(fmaxf(fmaxf(s[8 * c], s[8 * c + 1]), fmaxf(s[8 * c + 2], s[8 * c + 3])),
                          fmaxf(fmaxf(s[8 * c + 4], s[8 * c + 5]), fmaxf(s[8 * c + 6], s[8 * c + 7])));
          }
          mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * sc;
        }
        const float mt = fmaxf(mx, xchg(mx));
        // bf16: refresh the max only when it grows by more than 15 (p <= 2^15 fits
        // fp16); e4m3: p * 448 must stay within e4m3, so the exact running max
        const bool need = kFP8 ? (mt > m_run) : (mt > m_run + 15.0f);
        if (__any_sync(0xffffffffu, need)) {
          const float m_new = need ? mt : m_run;
          const float f = need ? ex2_approx(m_run - m_new) : 1.0f;
          if (i > 0) {
            // O holds P V of the previous steps: wait for the last PV, rescale
            ok = ok && warp_wait(&bars[B_PEMPTY + ((g - 1) & 1)], ((g - 1) >> 1) & 1, abort_flag, a.status, a.wait_ns);
            if (ok) {
              tc_fence_after();
#pragma unroll 1
              for (int cc = 0; cc < 4; ++cc) {  // 16 columns at a time
                float o[16];
                tmem_ld16(tmem + lrow + T_O + 64 * half + 16 * cc, o);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 16; ++c) o[c] *= f;
                tmem_st16f(tmem + lrow + T_O + 64 * half + 16 * cc, o);
              }
              tmem_wait_st();
            }
          }
          l_part *= f;
          m_run = m_new;
        }
        // pass 2: p = 2^(s*sc - m), 32 keys at a time; P goes over the first 32
        // (bf16) / 16 (e4m3) columns of this half's S, which pass 1 has read
        const float nm = -m_run;
        float l4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (live) {
#pragma unroll 1
          for (int cc = 0; cc < 2; ++cc) {
            float sk[32];
            tmem_ld32(scol + 32 * cc, sk);
            tmem_wait_ld();
            if constexpr (kI8) {
#pragma unroll
              for (int c = 0; c < 32; ++c) sk[c] = static_cast<float>(__float_as_int(sk[c]));
            }
            if (nvalid < kBlockKV) {
#pragma unroll
              for (int c = 0; c < 32; ++c)
                if (32 * cc + c >= nvalid) sk[c] = -INFINITY;
            }
            if constexpr (kFP8) {
              // the row sum uses the unquantised p; the PV product p * 448 rounded
              // to e4m3 (four keys per TMEM column)
              uint32_t pk[8];
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                float p[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) p[e] = ex2_approx(fmaf(sk[4 * c + e], sc, nm));
                l4[c & 3] += (p[0] + p[1]) + (p[2] + p[3]);
                const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(p[0] * 448.0f, p[1] * 448.0f),
                                                             __NV_SATFINITE, __NV_E4M3);
                const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(p[2] * 448.0f, p[3] * 448.0f),
                                                             __NV_SATFINITE, __NV_E4M3);
                pk[c] = lo | (hi << 16);
              }
              tmem_st8(scol + 8 * cc, pk);
            } else {
              uint32_t pk[16];
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const float p0 = ex2_approx(fmaf(sk[2 * c], sc, nm));
                const float p1 = ex2_approx(fmaf(sk[2 * c + 1], sc, nm));
                l4[c & 3] += p0 + p1;
                pk[c] = pack_half2(p0, p1);
              }
              tmem_st16(scol + 16 * cc, pk);
            }
          }
        }
        l_part += (l4[0] + l4[1]) + (l4[2] + l4[3]);
        if (ok) {
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&bars[B_PFULL + b]);
        }
        if (i == 0) release_store();
        zex += zv;
      }
      gs += T.nsteps;
      // SLA: the negligible blocks only leave the linear sum
      if (T.has_lin) {
        float z4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int it = T.n_crit + half; it < T.n_total; it += 8) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i2 = it + 2 * u;
            if (i2 < T.n_total) z4[u] += zb[static_cast<long long>(block_at(T, i2, a.nkv, nullptr)) * kDPad];
          }
        }
        zex += (z4[0] + z4[1]) + (z4[2] + z4[3]);
      }

      // ---------------------------------------------------------- epilogue
      // Work that needs no product first (l, Z_i and the denominator), then H_i
      // once warp 10's products are done, then phi(Q) over the last S buffer once
      // the last PV has read it.
      release_store();  // (a tile without steps)
      const float l_run = l_part + xchg(l_part);
      const uint32_t pcol = T_S0 + ((gs - 1) & 1) * 128;  // the tile's last S buffer
      const int hidx = gv + T.nsteps + T.nnegl_e;          // value entry of the H tile
      const int hsl = hidx % kVSlots;
      uint8_t* hbuf = sm + OFF_V + hsl * VSLOT;
      gv += T.nsteps + T.nnegl_e + (T.has_lin ? 1 : 0);
      float den = 0.0f;
      if (T.has_lin) {
        // Z_i[e] for e = r, shared with every row for the denominator
        const float zi = zt_r - (zex + xchg(zex));
        if (half == 0) zsh[r] = zi;
        const int c0 = 64 * half;
        named_bar_sync(5, kCompute);  // Z_i complete
        float dp = 0.0f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float2 f = unpack_half2(phq[c]);  // the denominator uses the rounded phi(Q)
          dp = fmaf(f.x, zsh[c0 + 2 * c], dp);
          dp = fmaf(f.y, zsh[c0 + 2 * c + 1], dp);
        }
        den = dp + xchg(dp);
        ok = ok && warp_wait(&bars[B_HFIN], ti & 1, abort_flag, a.status, a.wait_ns);
        if (ok) tc_fence_after();
        // H_i / sigma = H_tot / sigma (fp16 tile from TMA) - H_ex / sigma, row e = r,
        // channels 64*half.., in place in the MN-major H tile
        ok = ok && warp_wait(&bars[B_VFULL + hsl], (hidx / kVSlots) & 1, abort_flag, a.status, a.wait_ns);
        const float inv_sigma = 1.0f / sigma;  // exact: sigma is a power of two
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float hk[32];
          tmem_ld32(tmem + lrow + T_HK + 64 * half + 32 * cc, hk);  // stale without listed blocks: dropped below
          tmem_wait_ld();
          const bool use_h = ok && T.n_total > 0;
#pragma unroll
          for (int c = 0; c < 32; ++c) hk[c] = use_h ? hk[c] : 0.0f;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4* hp = reinterpret_cast<uint4*>(hbuf + half * 16384u + sw128_off(r, 4 * cc + q4));
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
      } else {
        ok = ok && warp_wait(&bars[B_HFIN], ti & 1, abort_flag, a.status, a.wait_ns);  // (every tile: phases stay aligned)
      }
      ok = ok && warp_wait(&bars[B_OFINAL], ti & 1, abort_flag, a.status, a.wait_ns);
      if (ok) tc_fence_after();
      if (T.has_lin) {
        if (ok) {
          tmem_st16(tmem + lrow + pcol + 32 * half, phq);
          tmem_st16(tmem + lrow + pcol + 32 * half + 16, phq + 16);
          tmem_wait_st();
        }
        fence_proxy_async_smem();  // the H_i tile is visible to the tensor core
      }
      if (ok) {
        tc_fence_before();
        mbar_arrive(&bars[B_EPI]);
      }
      // the next tile's phi(Q) while phi(Q) H_i runs
      if (t + static_cast<int>(gridDim.x) < ntiles) form_phi_q(tile_at(a, t + gridDim.x, false), ti + 1);
      ok = ok && warp_wait(&bars[B_NUM], ti & 1, abort_flag, a.status, a.wait_ns);
      if (ok) tc_fence_after();

      const float inv_l = (T.n_crit > 0 && l_run > 0.0f) ? 1.0f / l_run : 0.0f;
      const float lin_scale = (T.has_lin && den > 0.0f) ? sigma / den : 0.0f;
      float w_s, lin_w;
      if (a.wproj != nullptr) {
        w_s = inv_l;
        lin_w = 1.0f;
        if (T.has_lin) {
          // SLA: O_l -> bf16 hi + lo into TMEM (A operand), W_proj -> the H tile's slot (MN-major)
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            float ol[32];
            if (ok) {
              tmem_ld32(tmem + lrow + T_HK + 64 * half + 32 * cc, ol);
              tmem_wait_ld();
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c) ol[c] = 0.0f;
            }
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float v0 = ol[2 * c] * lin_scale, v1 = ol[2 * c + 1] * lin_scale;
              hi[c] = pack_bf162(v0, v1);
              const float2 hb = unpack_bf162(hi[c]);
              lo[c] = pack_bf162(v0 - hb.x, v1 - hb.y);
            }
            if (ok) {
              tmem_st16(tmem + lrow + pcol + 32 * half + 16 * cc, hi);
              tmem_st16(tmem + lrow + pcol + 64 + 32 * half + 16 * cc, lo);
            }
          }
          const __nv_bfloat16* wp = static_cast<const __nv_bfloat16*>(a.wproj);
          for (int idx = tid; idx < 128 * 16; idx += kCompute) {
            const int e = idx >> 4, u = idx & 15;
            uint4 w = make_uint4(0, 0, 0, 0);
            if (e < a.d && 8 * u < a.d) w = *reinterpret_cast<const uint4*>(wp + e * a.d + 8 * u);
            *reinterpret_cast<uint4*>(hbuf + (u >> 3) * 16384u + sw128_off(e, u & 7)) = w;
          }
          if (ok) tmem_wait_st();
          fence_proxy_async_smem();
        }
        if (ok) {
          tc_fence_before();
          mbar_arrive(&bars[B_PROJR]);
        }
        ok = ok && warp_wait(&bars[B_PROJF], ti & 1, abort_flag, a.status, a.wait_ns);
        if (ok) tc_fence_after();
      } else {
        w_s = alpha_t * inv_l;
        lin_w = (1.0f - alpha_t) * lin_scale;
      }
      // combine 32 channels at a time; TMEM goes back after the last read.  With
      // a TMA store the bf16 rows are staged in the H tile's slot (its products
      // are done) and leave as two 64-channel boxes.
      const bool tma_o = a.tma_out && T.has_lin;
      const long long obase = (static_cast<long long>(T.bh) * a.N + tok) * a.d;
      float bs = 0.0f, bl = 0.0f;  // backward statistics: dO . O_s, dO . O_l over this half's channels
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int ch0 = 64 * half + 32 * cc;
        // both accumulators are read unconditionally (a stale column is dropped by the select below)
        float o[32], nmv[32];
        tmem_ld32(tmem + lrow + T_O + ch0, o);
        tmem_ld32(tmem + lrow + T_HK + ch0, nmv);
        tmem_wait_ld();
        if (cc == 1 && ok) {
          tc_fence_before();
          mbar_arrive(&bars[B_EPIDONE]);
        }
        if constexpr (kFP8) {  // O accumulates e4m3 codes: times (absmax_c / 448) / 448 per channel
          const float* va = a.vamax + static_cast<long long>(T.bh) * kDPad + ch0;
#pragma unroll
          for (int c = 0; c < 32; ++c)
            o[c] *= __fdiv_rn(va[c] > 0.0f ? __fdiv_rn(va[c], 448.0f) : __fdiv_rn(1.0f, 448.0f), 448.0f);
        }
        const bool use_s = ok && T.n_crit > 0, use_l = ok && T.has_lin;
        if constexpr (kStats && !kFP8) {
          if (row_valid) {
            const __nv_bfloat16* gp = static_cast<const __nv_bfloat16*>(a.bwd_do) + obase + ch0;
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              const uint4 w = *reinterpret_cast<const uint4*>(gp + 8 * q8);
              const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 g2 = unpack_bf162(ww[e]);
                const int c = 8 * q8 + 2 * e;
                bs = fmaf(g2.x, use_s ? o[c] * inv_l : 0.0f, bs);
                bs = fmaf(g2.y, use_s ? o[c + 1] * inv_l : 0.0f, bs);
                bl = fmaf(g2.x, use_l ? nmv[c] * lin_scale : 0.0f, bl);
                bl = fmaf(g2.y, use_l ? nmv[c + 1] * lin_scale : 0.0f, bl);
              }
            }
          }
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float os = use_s ? o[c] * w_s : 0.0f;
          const float olv = use_l ? nmv[c] * lin_w : 0.0f;
          o[c] = os + olv;
        }
        if (tma_o) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8)
            *reinterpret_cast<uint4*>(hbuf + half * 16384u + sw128_off(r, 4 * cc + q8)) =
                make_uint4(pack_bf162(o[8 * q8], o[8 * q8 + 1]), pack_bf162(o[8 * q8 + 2], o[8 * q8 + 3]),
                           pack_bf162(o[8 * q8 + 4], o[8 * q8 + 5]), pack_bf162(o[8 * q8 + 6], o[8 * q8 + 7]));
        } else if (ok && row_valid && (!kStats || a.out != nullptr)) {
          if (a.out_bf16) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + obase;
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8)
              if (ch0 + 8 * q8 < a.d)
                *reinterpret_cast<uint4*>(dst + ch0 + 8 * q8) =
                    make_uint4(pack_bf162(o[8 * q8], o[8 * q8 + 1]), pack_bf162(o[8 * q8 + 2], o[8 * q8 + 3]),
                               pack_bf162(o[8 * q8 + 4], o[8 * q8 + 5]), pack_bf162(o[8 * q8 + 6], o[8 * q8 + 7]));
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
      if constexpr (kStats) {
        bs += xchg(bs);
        bl += xchg(bl);
        if (half == 0 && row_valid) {
          const bool lin = T.has_lin && den > 0.0f;
          float4* rp = reinterpret_cast<float4*>(a.bwd_rows + (static_cast<long long>(T.bh) * a.N + tok) * 8);
          rp[0] = make_float4((T.n_crit > 0 && l_run > 0.0f) ? m_run + log2f(l_run) : 0.0f, alpha_t * bs,
                              lin ? (1.0f - alpha_t) / den : 0.0f, lin ? -(1.0f - alpha_t) * bl / den : 0.0f);
          rp[1] = make_float4(bs - bl, 0.0f, 0.0f, 0.0f);
        }
      }
      if (tma_o) {
        fence_proxy_async_smem();      // the staged rows are visible to the TMA engine
        named_bar_sync(5, kCompute);   // ... from every thread
        if (tid == 0 && ok) {
          tma_store_3d(&tmO, hbuf, 0, T.qb * 128, T.bh);
          tma_store_3d(&tmO, hbuf + 16384, 64, T.qb * 128, T.bh);
          bulk_commit_group();
        }
        pend_store = true;  // the slot is refilled once the store has read it (release_store)
        pend_hsl = hsl;
      }
    }
    if (tid == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

template <int kLow, bool kStats = false>
static cudaError_t launch_sparse_t(const SparseArgs& a, const CUtensorMap& mq, const CUtensorMap& mk,
                                   const CUtensorMap& mp, const CUtensorMap& mv, const CUtensorMap& mh,
                                   const CUtensorMap& mv8, const CUtensorMap& mo, cudaStream_t st) {
  constexpr uint32_t smem = Lay<kLow != 0>::SMEM_BYTES;
  cudaError_t e =
      cudaFuncSetAttribute(sparse_fwd_kernel<kLow, kStats>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = kNumSMs;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long ntiles = static_cast<long long>(a.BH) * a.nq;
  const unsigned grid = static_cast<unsigned>(ntiles < sms ? ntiles : sms);
  sparse_fwd_kernel<kLow, kStats><<<grid, kThreads, smem, st>>>(mq, mk, mp, mv, mh, mv8, mo, a);
  return cudaGetLastError();
}

cudaError_t launch_sparse(const SparseArgs& a_in, const void* q_bf16_128, const void* k_bf16_128,
                          const void* phik16, const void* v16, const void* hs16, const void* q8, const void* k8,
                          const void* v8, cudaStream_t st) {
  CUtensorMap mq, mk, mp, mv, mh, mv8, mo;
  cudaError_t e;
  SparseArgs a = a_in;
  // bf16 output of 128-row query blocks at d = 128 leaves through TMA tile stores
  a.tma_out = (a.out_bf16 && a.d == kDPad && a.bq == 128) ? 1 : 0;
  if (a.tma_out) {
    if ((e = encode_map(&mo, a.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.N, a.BH, 128)) != cudaSuccess) return e;
  } else {
    mo = {};
  }
  if ((e = encode_map(&mp, phik16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.N, a.BH, 64)) != cudaSuccess) return e;
  if ((e = encode_map(&mv, v16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.N, a.BH, 64)) != cudaSuccess) return e;
  if ((e = encode_map(&mh, hs16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, kDPad, a.BH, 128)) != cudaSuccess) return e;
  if (a.fp8) {
    if ((e = encode_map8(&mq, q8, a.N, a.BH, 128)) != cudaSuccess) return e;
    if ((e = encode_map8(&mk, k8, a.N, a.BH, 64)) != cudaSuccess) return e;
    if ((e = encode_map8(&mv8, v8, a.N, a.BH, 64)) != cudaSuccess) return e;
    if (a.fp8 == 2) return launch_sparse_t<2>(a, mq, mk, mp, mv, mh, mv8, mo, st);
    return launch_sparse_t<1>(a, mq, mk, mp, mv, mh, mv8, mo, st);
  }
  if ((e = encode_map(&mq, q_bf16_128, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.N, a.BH, 128)) != cudaSuccess) return e;
  if ((e = encode_map(&mk, k_bf16_128, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.N, a.BH, 64)) != cudaSuccess) return e;
  if (a.bwd_rows != nullptr) return launch_sparse_t<0, true>(a, mq, mk, mp, mv, mh, mv, mo, st);
  return launch_sparse_t<0>(a, mq, mk, mp, mv, mh, mv, mo, st);
}

}  // namespace sla
