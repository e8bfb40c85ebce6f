// prepare.cu -- linear-branch totals and the operand staging of the attention
// kernel.
//
// "SLA: Beyond Sparsity in Diffusion Transformers …" (papernotes.org) 关键设计 3
// defines the linear branch through H_i = sum_j phi(K_j)^T V_j and
// Z_i = sum_j colsum phi(K_j) over the marginal blocks; 关键设计 4 precomputes
// the per-block h_j, z_j.  Here the totals over all N tokens are formed once
// per (b,h); the attention kernel subtracts the blocks it does not treat
// linearly.  "SLA2 深度解读 …" (jefxiong.cn) §08 describes the same aggregation
// of (K^phi)^T V for the blocks the mask misses.
//
// lin_prepass_kernel: per (b,h) and a contiguous range of 64-token key blocks,
//   phi(K) -> fp16 and V -> fp16 (written to the workspace for the attention
//   kernel, channels past d zero), and the partial sums
//   H_part = phi(K)^T V (tcgen05, fp16 in / fp32 accumulate in TMEM) and
//   Z_part = phi(K)^T 1 (same, against a column of ones).
// zsum_kernel / hsum_kernel: Z_tot, H_tot = sum of the partials in split
//   order (fixed, so deterministic); H_tot is stored as fp16 H_tot / sigma
//   with sigma an exact per-head power of two (see hsum_kernel).
// lin_prepass_tma_kernel (bf16, d = 128) also writes the router's key-block
//   means ("SLA2 深度解读 …" §05: pool(K)) while each key block sits in shared
//   memory, so the router need not read K again (SLA_ROUTE_KBAR_FROM_WS).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "sla_device.cuh"
#include "sla_internal.h"
#include "sla_kernels.h"

namespace sla {

namespace {

constexpr int kPreThreads = 256;
constexpr int kUnits = 64 * 16 / kPreThreads;  // 16-byte channel units per thread per 64-token tile
constexpr uint32_t kTileBytes = 64 * 128 * 2;  // 64 tokens x 128 channels x 2 B
constexpr uint32_t kOffPhi0 = 0;
constexpr uint32_t kOffV0 = kTileBytes;
constexpr uint32_t kBufBytes = 2 * kTileBytes;       // phi(K) + V for one buffer
constexpr uint32_t kOffOnes = 2 * kBufBytes;          // 65536
constexpr uint32_t kOffBar = kOffOnes + 2048;         // 2 mma barriers + done
constexpr uint32_t kOffMisc = kOffBar + 64;           // tmem base, abort flag
constexpr uint32_t kOffZred = kOffMisc + 64;          // [2][8 warps][128] column partials
constexpr uint32_t kPreSmem = kOffZred + 2 * 8 * 128 * 4 + 1024;  // + alignment slack
constexpr uint32_t kPreTmemCols = 128;                // H: 0..127

// Raw 16-byte words holding 8 consecutive channels of T.
template <typename T>
struct Raw8 {
  static constexpr int W = sizeof(T) * 8 / 16;  // 1 for bf16, 2 for f32
  uint4 w[W];
};

template <typename T>
__device__ __forceinline__ void load_raw8(const T* __restrict__ base, long long row, int d, int u, bool valid,
                                          Raw8<T>& r) {
#pragma unroll
  for (int i = 0; i < Raw8<T>::W; ++i) r.w[i] = make_uint4(0, 0, 0, 0);
  if (!valid || 8 * u >= d) return;
  const uint4* src = reinterpret_cast<const uint4*>(base + row * d + 8 * u);
#pragma unroll
  for (int i = 0; i < Raw8<T>::W; ++i) r.w[i] = __ldg(src + i);
}

template <typename T>
__device__ __forceinline__ void unpack8(const Raw8<T>& r, float* f) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t w[4] = {r.w[0].x, r.w[0].y, r.w[0].z, r.w[0].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 p = unpack_bf162(w[i]);
      f[2 * i] = p.x;
      f[2 * i + 1] = p.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      f[4 * i + 0] = __uint_as_float(r.w[i].x);
      f[4 * i + 1] = __uint_as_float(r.w[i].y);
      f[4 * i + 2] = __uint_as_float(r.w[i].z);
      f[4 * i + 3] = __uint_as_float(r.w[i].w);
    }
  }
}

// 8 consecutive channels [8u, 8u+8) of token row `row` as fp32; zero past d.
template <typename T>
__device__ __forceinline__ void load8(const T* __restrict__ base, long long row, int d, int u, bool valid,
                                      float* f) {
  Raw8<T> r;
  load_raw8<T>(base, row, d, u, valid, r);
  unpack8<T>(r, f);
}

template <typename T>
__global__ void __launch_bounds__(kPreThreads, 2) lin_prepass_kernel(
    const T* __restrict__ k, const T* __restrict__ v, __half* __restrict__ phik, __half* __restrict__ v16,
    __nv_bfloat16* __restrict__ khat, float* __restrict__ hpart, float* __restrict__ zpart,
    float* __restrict__ zblk, float* __restrict__ kstat, float* __restrict__ vstat, int N, int d, int nkv,
    int nsplit, int phi_kind, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(sm + kOffBar);  // [0], [1]
  uint64_t* done_bar = mma_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kOffMisc + 4);
  float* zred = reinterpret_cast<float*>(sm + kOffZred);

  const int tid = threadIdx.x, warp = tid / 32;
  const int split = blockIdx.x;
  const long long bh = blockIdx.y;
  const int jb0 = static_cast<int>((static_cast<long long>(split) * nkv) / nsplit);
  const int jb1 = static_cast<int>((static_cast<long long>(split + 1) * nkv) / nsplit);

  if (tid == 0) {
    mbar_init(&mma_bar[0], 1);
    mbar_init(&mma_bar[1], 1);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kPreTmemCols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const T* kb = k + bh * static_cast<long long>(N) * d;
  const T* vb = v + bh * static_cast<long long>(N) * d;
  __half* phib = phik + bh * static_cast<long long>(N) * kDPad;
  __half* v16b = v16 + bh * static_cast<long long>(N) * kDPad;
  __nv_bfloat16* khb = khat ? khat + bh * static_cast<long long>(N) * kDPad : nullptr;

  const uint32_t idesc_h = idesc_f16(0, 1, 1, 128, 128);  // phi(K)^T (MN-major) x V (MN-major)
  bool ok = true;
  float zacc = 0.0f;  // threads < 128: this split's Z for channel tid, blocks in ascending order
  float ksum[8], vmax[8];  // this thread's channels [8u, 8u+8): sum of K, absmax of V over its rows
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    ksum[e] = 0.0f;
    vmax[e] = 0.0f;
  }

  // this thread's units of a 64-token tile: row m = tid/16 + 16*i, channels [8u, 8u+8)
  const int u = tid % 16;
  Raw8<T> kr[kUnits], vr[kUnits];
  auto fetch = [&](int jb) {
#pragma unroll
    for (int i = 0; i < kUnits; ++i) {
      const int tok = jb * 64 + tid / 16 + 16 * i;
      load_raw8<T>(kb, tok, d, u, tok < N, kr[i]);
      load_raw8<T>(vb, tok, d, u, tok < N, vr[i]);
    }
  };
  if (jb0 < jb1) fetch(jb0);

  for (int jb = jb0; jb < jb1; ++jb) {
    const int it = jb - jb0;
    const int buf = it & 1;
    uint8_t* sphi = sm + buf * kBufBytes + kOffPhi0;
    uint8_t* sv = sm + buf * kBufBytes + kOffV0;
    float kf[kUnits][8], vf[kUnits][8];
#pragma unroll
    for (int i = 0; i < kUnits; ++i) {
      unpack8<T>(kr[i], kf[i]);
      unpack8<T>(vr[i], vf[i]);
#pragma unroll
      for (int e = 0; e < 8; ++e) {  // rows past N hold zeros
        ksum[e] += kf[i][e];
        vmax[e] = fmaxf(vmax[e], fabsf(vf[i][e]));
      }
    }
    if (jb + 1 < jb1) fetch(jb + 1);  // next tile's loads overlap this tile's work
    // buffer reuse: the MMA that read this buffer two tiles ago must be done
    if (it >= 2) {
      if (!mbar_wait(&mma_bar[buf], ((it - 2) >> 1) & 1, abort_flag, status)) ok = false;
    }
    ok = __syncthreads_and(ok) != 0;  // CTA-uniform verdict
    if (!ok) break;
    float csum[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};  // this thread's rows, rounded phi(K)
#pragma unroll
    for (int i = 0; i < kUnits; ++i) {
      const int m = tid / 16 + 16 * i;
      const int tok = jb * 64 + m;
      const bool valid = tok < N;
      float ph[8];
      if (phi_kind == SLA_PHI_SOFTMAX) {
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (8 * u + e < d) mx = fmaxf(mx, kf[i][e]);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float v = ex2_approx((kf[i][e] - mx) * 1.4426950408889634f);  // evaluated, then selected
          ph[e] = (8 * u + e < d) ? v : 0.0f;
          sum += ph[e];
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float inv = 1.0f / sum;
#pragma unroll
        for (int e = 0; e < 8; ++e) ph[e] *= inv;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float v = elu1(kf[i][e]);  // evaluated, then selected: no branch
          ph[e] = (8 * u + e < d) ? v : 0.0f;
        }
      }
      uint4 pu, vu;
      if (valid) {
        pu = make_uint4(pack_half2(ph[0], ph[1]), pack_half2(ph[2], ph[3]), pack_half2(ph[4], ph[5]),
                        pack_half2(ph[6], ph[7]));
        vu = make_uint4(pack_half2(vf[i][0], vf[i][1]), pack_half2(vf[i][2], vf[i][3]),
                        pack_half2(vf[i][4], vf[i][5]), pack_half2(vf[i][6], vf[i][7]));
        const uint32_t pw[4] = {pu.x, pu.y, pu.z, pu.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack_half2(pw[e]);
          csum[2 * e] += f.x;
          csum[2 * e + 1] += f.y;
        }
        const long long g = static_cast<long long>(tok) * kDPad + 8 * u;
        *reinterpret_cast<uint4*>(phib + g) = pu;
        *reinterpret_cast<uint4*>(v16b + g) = vu;
        if (khb) {
          const uint4 ku = make_uint4(pack_bf162(kf[i][0], kf[i][1]), pack_bf162(kf[i][2], kf[i][3]),
                                      pack_bf162(kf[i][4], kf[i][5]), pack_bf162(kf[i][6], kf[i][7]));
          *reinterpret_cast<uint4*>(khb + g) = ku;
        }
      } else {
        pu = make_uint4(0, 0, 0, 0);
        vu = pu;
      }
      const uint32_t off = (u >> 3) * 8192u + sw128_off(m, u & 7);
      *reinterpret_cast<uint4*>(sphi + off) = pu;
      *reinterpret_cast<uint4*>(sv + off) = vu;
    }
    // column sums of this key block: lanes u and u+16 hold the same channels
#pragma unroll
    for (int e = 0; e < 8; ++e) csum[e] += __shfl_xor_sync(0xffffffffu, csum[e], 16);
    if ((tid & 31) < 16) {
#pragma unroll
      for (int e = 0; e < 8; ++e) zred[warp * 128 + 8 * u + e] = csum[e];
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid < 128) {
      float z = 0.0f;
#pragma unroll
      for (int w = 0; w < kPreThreads / 32; ++w) z += zred[w * 128 + tid];
      zblk[(bh * nkv + jb) * kDPad + tid] = z;
      zacc += z;
    }
    if (tid == 0) {
      tc_fence_after();
      const uint32_t aphi = smem_u32(sphi), av = smem_u32(sv);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t a = sdesc_sw128(aphi + kk * 2048, 8192, 1024);
        const uint64_t b = sdesc_sw128(av + kk * 2048, 8192, 1024);
        const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
        mma_f16_ss(tmem + 0, a, b, idesc_h, acc);
      }
      mma_commit(&mma_bar[buf]);
    }
  }
  // all MMAs of this CTA done -> read the partial sums out of TMEM (warps 0..3: one lane each)
  if (tid == 0) mma_commit(done_bar);
  __syncwarp();
  bool have = ok && (jb1 > jb0);
  {
    // warp-uniform wait: lane 0 waits, the warp follows its verdict
    int w_ok = 0;
    if ((tid & 31) == 0) w_ok = mbar_wait(done_bar, 0, abort_flag, status) ? 1 : 0;
    w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
    have = have && w_ok;
  }
  tc_fence_after();
  // per-split K column sums and V column absmax (used by the low-bit branch)
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    ksum[e] += __shfl_xor_sync(0xffffffffu, ksum[e], 16);
    vmax[e] = fmaxf(vmax[e], __shfl_xor_sync(0xffffffffu, vmax[e], 16));
  }
  __syncthreads();  // zred free
  float* kred = reinterpret_cast<float*>(sm + kOffZred);
  float* vred = kred + 8 * 128;
  if ((tid & 31) < 16) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      kred[warp * 128 + 8 * u + e] = ksum[e];
      vred[warp * 128 + 8 * u + e] = vmax[e];
    }
  }
  __syncthreads();
  if (tid < 128) {
    float ks = 0.0f, vm = 0.0f;
#pragma unroll
    for (int w = 0; w < kPreThreads / 32; ++w) {
      ks += kred[w * 128 + tid];
      vm = fmaxf(vm, vred[w * 128 + tid]);
    }
    kstat[(bh * nsplit + split) * kDPad + tid] = ks;
    vstat[(bh * nsplit + split) * kDPad + tid] = vm;
  }
  if (have && warp < 4) {
    zpart[(bh * nsplit + split) * kDPad + tid] = zacc;
    float* hp = hpart + ((bh * nsplit + split) * kDPad + tid) * kDPad;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      float x[32];
      tmem_ld32(tmem + ((warp * 32) << 16) + cc * 32, x);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4*>(hp + cc * 32 + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kPreTmemCols);
  }
}

// lin_prepass_tma_kernel: the same results for bf16 inputs with d = 128 (the
// video shapes), built for HBM throughput.  K and V tiles (64 tokens) arrive
// by TMA in a kStagesP-deep ring; the threads turn them into phi(K) and V as
// fp16 in place (the 128-byte swizzled layout of the load is the layout the
// tensor core reads); a TMA tile store writes them to the workspace and the
// same tiles feed H_part += phi(K)^T V.  A stage is refilled once its product
// is done and its store has read it.  Thread 0 issues every TMA operation and
// product; all waits are bounded.
constexpr int kStagesP = 3;
constexpr uint32_t kStageBytes = 2 * kTileBytes;  // K (-> phi(K)) | V (-> fp16)
constexpr uint32_t kTOffBar = kStagesP * kStageBytes;            // full[kStagesP], mma[kStagesP], done
constexpr uint32_t kTOffMisc = kTOffBar + 128;                   // tmem base, abort flag
constexpr uint32_t kTOffZred = kTOffMisc + 64;                   // [8 warps][128] column partials
constexpr uint32_t kTPreSmem = kTOffZred + 8 * 128 * 4;
static_assert(2 * kStagesP + 1 <= 16, "barrier area");

__global__ void __launch_bounds__(kPreThreads, 2) lin_prepass_tma_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __grid_constant__ CUtensorMap tmPhiOut, const __grid_constant__ CUtensorMap tmVOut,
    float* __restrict__ hpart, float* __restrict__ zpart, float* __restrict__ zblk, float* __restrict__ kstat,
    float* __restrict__ vstat, float* __restrict__ kbar, int N, int nkv, int nsplit, int phi_kind, int* status) {
  extern __shared__ __align__(1024) uint8_t sm[];
  if ((smem_u32(sm) & 1023u) != 0) {  // the swizzled tiles need a 1024-byte aligned window
    if (threadIdx.x == 0) report_error(status, SLA_ERR_UNSUPPORTED);
    return;
  }
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kTOffBar);
  uint64_t* mmad = full + kStagesP;
  uint64_t* done_bar = mmad + kStagesP;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kTOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kTOffMisc + 4);
  float* zred = reinterpret_cast<float*>(sm + kTOffZred);

  const int tid = threadIdx.x, warp = tid / 32;
  const int split = blockIdx.x;
  const int bh = blockIdx.y;
  const int jb0 = static_cast<int>((static_cast<long long>(split) * nkv) / nsplit);
  const int jb1 = static_cast<int>((static_cast<long long>(split + 1) * nkv) / nsplit);
  const int nt = jb1 - jb0;

  if (tid == 0) {
    for (int i = 0; i < kStagesP; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&mmad[i], 1);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kPreTmemCols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int issued = 0;  // thread 0: tiles whose loads were issued
  auto load_tile = [&](int it) {  // thread 0: tile it of this split into stage it % kStagesP
    issued = it + 1;
    uint8_t* st = sm + (it % kStagesP) * kStageBytes;
    uint64_t* fb = &full[it % kStagesP];
    const int row = (jb0 + it) * 64;
    mbar_arrive_expect_tx(fb, kStageBytes);
    tma_load_3d(st, &tmK, fb, 0, row, bh);
    tma_load_3d(st + 8192, &tmK, fb, 64, row, bh);
    tma_load_3d(st + kTileBytes, &tmV, fb, 0, row, bh);
    tma_load_3d(st + kTileBytes + 8192, &tmV, fb, 64, row, bh);
  };
  if (tid == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (int it = 0; it < kStagesP - 1 && it < nt; ++it) load_tile(it);
  }

  const uint32_t idesc_h = idesc_f16(0, 1, 1, 128, 128);  // phi(K)^T (MN-major) x V (MN-major)
  bool ok = true;
  float zacc = 0.0f;  // threads < 128: this split's Z for channel tid, blocks in ascending order
  float ksum[8], vmax[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    ksum[e] = 0.0f;
    vmax[e] = 0.0f;
  }
  const int u = tid % 16;  // this thread's 16-byte unit (channels 8u .. 8u+7) of rows tid/16 + 16 i
  for (int it = 0; it < nt; ++it) {
    const int jb = jb0 + it;
    const int stg = it % kStagesP;
    uint8_t* sk = sm + stg * kStageBytes;
    uint8_t* sv = sk + kTileBytes;
    ok = ok && mbar_wait(&full[stg], (it / kStagesP) & 1, abort_flag, status);
    ok = __syncthreads_and(ok) != 0;  // CTA-uniform verdict
    if (!ok) break;
    {
      // The router's mean of key block jb [SLA2-deep §05], from the raw K tile
      // before it turns into phi(K) in place: channel tid, the block's tokens in
      // ascending order from +0.0 in fp32, then one division by their count
      // (the same arithmetic as the router's own pooling).
      if (tid < 128) {
        const int cnt = min(64, N - jb * 64);
        const uint32_t cb = (tid >> 6) * 8192u + ((tid & 7) << 1);
        const int u8 = (tid >> 3) & 7;
        float acc = 0.0f;
#pragma unroll 8
        for (int t = 0; t < cnt; ++t)
          acc = __fadd_rn(acc, __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sk + cb + sw128_off(t, u8))));
        kbar[(static_cast<long long>(bh) * nkv + jb) * 128 + tid] = __fdiv_rn(acc, static_cast<float>(cnt));
      }
      __syncthreads();  // every column is summed before the tile is converted
    }
    float csum[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};  // this thread's rows, rounded phi(K)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = tid / 16 + 16 * i;
      const bool valid = jb * 64 + m < N;
      const uint32_t off = (u >> 3) * 8192u + sw128_off(m, u & 7);
      uint4* kp = reinterpret_cast<uint4*>(sk + off);
      uint4* vp = reinterpret_cast<uint4*>(sv + off);
      const uint4 kw = *kp, vw = *vp;  // rows past N were zero-filled by the load
      float kf[8], vf[8];
      {
        const uint32_t a[4] = {kw.x, kw.y, kw.z, kw.w}, b[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 p = unpack_bf162(a[e]), q = unpack_bf162(b[e]);
          kf[2 * e] = p.x;
          kf[2 * e + 1] = p.y;
          vf[2 * e] = q.x;
          vf[2 * e + 1] = q.y;
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        ksum[e] += kf[e];
        vmax[e] = fmaxf(vmax[e], fabsf(vf[e]));
      }
      float ph[8];
      if (phi_kind == SLA_PHI_SOFTMAX) {
        float mx = kf[0];
#pragma unroll
        for (int e = 1; e < 8; ++e) mx = fmaxf(mx, kf[e]);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          ph[e] = ex2_approx((kf[e] - mx) * 1.4426950408889634f);
          sum += ph[e];
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float inv = 1.0f / sum;
#pragma unroll
        for (int e = 0; e < 8; ++e) ph[e] *= inv;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) ph[e] = elu1(kf[e]);
      }
      uint4 pu = make_uint4(pack_half2(ph[0], ph[1]), pack_half2(ph[2], ph[3]), pack_half2(ph[4], ph[5]),
                            pack_half2(ph[6], ph[7]));
      const uint4 vu = make_uint4(pack_half2(vf[0], vf[1]), pack_half2(vf[2], vf[3]), pack_half2(vf[4], vf[5]),
                                  pack_half2(vf[6], vf[7]));
      if (!valid) pu = make_uint4(0, 0, 0, 0);  // keys past N leave the sums (V is zero there)
      const uint32_t pw[4] = {pu.x, pu.y, pu.z, pu.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack_half2(pw[e]);
        csum[2 * e] += f.x;
        csum[2 * e + 1] += f.y;
      }
      *kp = pu;
      *vp = vu;
    }
    // column sums of this key block: lanes u and u+16 hold the same channels
#pragma unroll
    for (int e = 0; e < 8; ++e) csum[e] += __shfl_xor_sync(0xffffffffu, csum[e], 16);
    if ((tid & 31) < 16) {
#pragma unroll
      for (int e = 0; e < 8; ++e) zred[warp * 128 + 8 * u + e] = csum[e];
    }
    fence_proxy_async_smem();  // the fp16 tiles are visible to the TMA store and the tensor core
    tc_fence_before();
    __syncthreads();
    if (tid < 128) {
      float z = 0.0f;
#pragma unroll
      for (int w = 0; w < kPreThreads / 32; ++w) z += zred[w * 128 + tid];
      zblk[(static_cast<long long>(bh) * nkv + jb) * kDPad + tid] = z;
      zacc += z;
    }
    if (tid == 0) {
      tc_fence_after();
      // phi(K), V (fp16) to the workspace (rows past N are not written)
      tma_store_3d(&tmPhiOut, sk, 0, jb * 64, bh);
      tma_store_3d(&tmPhiOut, sk + 8192, 64, jb * 64, bh);
      tma_store_3d(&tmVOut, sv, 0, jb * 64, bh);
      tma_store_3d(&tmVOut, sv + 8192, 64, jb * 64, bh);
      bulk_commit_group();
      const uint32_t aphi = smem_u32(sk), av = smem_u32(sv);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t a = sdesc_sw128(aphi + kk * 2048, 8192, 1024);
        const uint64_t b = sdesc_sw128(av + kk * 2048, 8192, 1024);
        mma_f16_ss(tmem + 0, a, b, idesc_h, (it > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(&mmad[stg]);
      // refill the stage of the previous tile: its product and its store must be done with it
      const int nx = it + kStagesP - 1;
      if (nx < nt) {
        if (it >= 1) {
          if (!mbar_wait(&mmad[(it - 1) % kStagesP], ((it - 1) / kStagesP) & 1, abort_flag, status)) ok = false;
          bulk_wait_read_one();  // all but the latest store group have read their tiles
        }
        if (ok) load_tile(nx);
      }
    }
    __syncthreads();  // zred is rewritten by the next tile
  }
  // all products done -> read the partial sums out of TMEM (warps 0..3: one lane each)
  if (tid == 0) {
    mma_commit(done_bar);
    bulk_wait_all();  // the stores are complete before the CTA exits
    // loads still in flight after an early exit must land before shared memory is reused
    for (int t = issued > kStagesP ? issued - kStagesP : 0; t < issued; ++t)
      mbar_wait_drain(&full[t % kStagesP], (t / kStagesP) & 1);
  }
  __syncwarp();
  bool have = ok && (nt > 0);
  {
    int w_ok = 0;
    if ((tid & 31) == 0) w_ok = mbar_wait(done_bar, 0, abort_flag, status) ? 1 : 0;
    w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
    have = have && w_ok;
  }
  tc_fence_after();
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    ksum[e] += __shfl_xor_sync(0xffffffffu, ksum[e], 16);
    vmax[e] = fmaxf(vmax[e], __shfl_xor_sync(0xffffffffu, vmax[e], 16));
  }
  __syncthreads();
  float* kred = zred;
  float* vred = reinterpret_cast<float*>(sm);  // stage 0 is idle now: 4 KB for the V partials
  if ((tid & 31) < 16) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      kred[warp * 128 + 8 * u + e] = ksum[e];
      vred[warp * 128 + 8 * u + e] = vmax[e];
    }
  }
  __syncthreads();
  if (tid < 128) {
    float ks = 0.0f, vm = 0.0f;
#pragma unroll
    for (int w = 0; w < kPreThreads / 32; ++w) {
      ks += kred[w * 128 + tid];
      vm = fmaxf(vm, vred[w * 128 + tid]);
    }
    kstat[(static_cast<long long>(bh) * nsplit + split) * kDPad + tid] = ks;
    vstat[(static_cast<long long>(bh) * nsplit + split) * kDPad + tid] = vm;
  }
  if (have && warp < 4) {
    zpart[(static_cast<long long>(bh) * nsplit + split) * kDPad + tid] = zacc;
    float* hp = hpart + ((static_cast<long long>(bh) * nsplit + split) * kDPad + tid) * kDPad;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      float x[32];
      tmem_ld32(tmem + ((warp * 32) << 16) + cc * 32, x);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4*>(hp + cc * 32 + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kPreTmemCols);
  }
}

// Z_tot[bh][e] = sum over splits (ascending) of each split's sum of per-block
// column sums, and the per-head scale sigma = 2^ceil(log2(max_e Z_tot)) (one
// block of 128 threads per head).
__global__ void __launch_bounds__(128) zsum_kernel(const float* __restrict__ zpart, float* __restrict__ ztot,
                                                   float* __restrict__ sigma, int nsplit) {
  const long long bh = blockIdx.x;
  const int e = threadIdx.x;
  float z = 0.0f;
  for (int s = 0; s < nsplit; ++s) z += zpart[(bh * nsplit + s) * kDPad + e];
  ztot[bh * kDPad + e] = z;
  __shared__ float red[4];
  float m = z;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((e & 31) == 0) red[e >> 5] = m;
  __syncthreads();
  if (e == 0) {
    m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    int ex = 0;
    if (m > 0.0f) frexpf(m, &ex);  // m < 2^ex
    sigma[bh] = ldexpf(1.0f, ex);
  }
}

// H_tot / sigma as fp16: sum of H_part over splits in ascending order, then one
// exact power-of-two scaling and one rounding.  |H_tot / sigma| <= max |V|
// because phi(K) >= 0 makes H_tot[e][c] a phi-weighted sum of v[c] with
// total weight Z_tot[e] <= sigma.
__global__ void __launch_bounds__(256) hsum_kernel(const float* __restrict__ hpart, const float* __restrict__ sigma,
                                                   __half* __restrict__ hs16, int BH, int nsplit) {
  const long long per = kDPad * kDPad;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= per * BH) return;
  const long long bh = idx / per, r = idx % per;
  float acc = 0.0f;
  for (int s = 0; s < nsplit; ++s) acc += hpart[(bh * nsplit + s) * per + r];
  hs16[idx] = __float2half_rn(acc / sigma[bh]);
}

// Q as bf16 with the head dim padded to 128 (needed when d != 128 or the
// input is fp32).  One thread per 8 output channels.
template <typename T>
__global__ void __launch_bounds__(256) qhat_kernel(const T* __restrict__ q, __nv_bfloat16* __restrict__ qhat,
                                                   long long rows, int d) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= rows * 16) return;
  const long long row = idx / 16;
  const int u = static_cast<int>(idx % 16);
  float f[8];
  load8<T>(q, row, d, u, true, f);
  *reinterpret_cast<uint4*>(qhat + row * kDPad + 8 * u) =
      make_uint4(pack_bf162(f[0], f[1]), pack_bf162(f[2], f[3]), pack_bf162(f[4], f[5]), pack_bf162(f[6], f[7]));
}

// ---------------------------------------------------------------- low-bit branch
// "SLA2 深度解读 …" (jefxiong.cn) §07: Q, K, P, V quantised for the sparse
// branch, K smoothed by its column mean first.  Readings (the page fixes
// neither format nor granularity): e4m3, round to nearest even, saturating;
// Q and K - mean(K) with one scale per 128-token block, V one per channel;
// a block or channel with absmax a is multiplied by 448/a before rounding
// and carries the scale a/448.

// mean(K) and absmax(V) per (b,h) channel from the prepass's per-split partials.
__global__ void __launch_bounds__(128) fp8_stats_kernel(const float* __restrict__ kstat,
                                                        const float* __restrict__ vstat, float* __restrict__ mu,
                                                        float* __restrict__ vamax, int nsplit, int N) {
  const long long bh = blockIdx.x;
  const int c = threadIdx.x;
  float ks = 0.0f, vm = 0.0f;
  for (int sp = 0; sp < nsplit; ++sp) {
    ks += kstat[(bh * nsplit + sp) * kDPad + c];
    vm = fmaxf(vm, vstat[(bh * nsplit + sp) * kDPad + c]);
  }
  mu[bh * kDPad + c] = ks / static_cast<float>(N);
  vamax[bh * kDPad + c] = vm;
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// Four signed INT8 codes: rint(x) with ties to even, saturated to [-127, 127].
__device__ __forceinline__ uint32_t i8x4(float a, float b, float c, float d) {
  const float x[4] = {a, b, c, d};
  uint32_t w = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int q = max(-127, min(127, __float2int_rn(x[e])));
    w |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * e);
  }
  return w;
}

__device__ __forceinline__ float block_absmax(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = 0.0f;
#pragma unroll
  for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w]);
  return m;
}

// One 128-token block of one head per CTA (256 threads, 8 channel units each):
// 8-bit copies of Q and K - mean(K) with the block's scale (e4m3 codes of
// x * 448 / amax, or with kInt8 the INT8 codes of x * 127 / amax), and the e4m3
// copy of V with the per-channel scale.  Channels past d and rows past N stay
// zero.
template <typename T, bool kInt8>
__global__ void __launch_bounds__(256) fp8_quant_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                        const T* __restrict__ v, const float* __restrict__ mu,
                                                        const float* __restrict__ vamax, uint8_t* __restrict__ q8,
                                                        uint8_t* __restrict__ k8, uint8_t* __restrict__ v8,
                                                        float* __restrict__ sq, float* __restrict__ sk, int N, int d,
                                                        int nb128) {
  __shared__ float red[8];
  const int blk = blockIdx.x;
  const long long bh = blockIdx.y;
  const int tid = threadIdx.x, u = tid % 16;
  const long long base = bh * static_cast<long long>(N);
  float mc[8], vinv[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int c = 8 * u + e;
    mc[e] = c < d ? mu[bh * kDPad + c] : 0.0f;
    const float a = c < d ? vamax[bh * kDPad + c] : 0.0f;
    vinv[e] = a > 0.0f ? __fdiv_rn(448.0f, a) : 1.0f;
  }
  for (int which = 0; which < 3; ++which) {
    const T* src = which == 0 ? q : (which == 1 ? k : v);
    uint8_t* dst = which == 0 ? q8 : (which == 1 ? k8 : v8);
    float x[8][8];
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int tok = blk * 128 + tid / 16 + 16 * i;
      load8<T>(src + base * d, tok, d, u, tok < N, x[i]);
      if (which == 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[i][e] = (tok < N && 8 * u + e < d) ? __fsub_rn(x[i][e], mc[e]) : 0.0f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(x[i][e]));
    }
    float inv[8];
    if (which < 2) {
      const float qmax = kInt8 ? 127.0f : 448.0f;
      const float amax = block_absmax(am, red);
      const float sc = amax > 0.0f ? __fdiv_rn(amax, qmax) : __fdiv_rn(1.0f, qmax);
      const float iv = amax > 0.0f ? __fdiv_rn(qmax, amax) : 1.0f;
      if (tid == 0) (which == 0 ? sq : sk)[bh * nb128 + blk] = sc;
#pragma unroll
      for (int e = 0; e < 8; ++e) inv[e] = iv;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) inv[e] = vinv[e];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int tok = blk * 128 + tid / 16 + 16 * i;
      if (tok < N) {
        const float* y = x[i];
        if (kInt8 && which < 2) {
          const uint2 w = make_uint2(i8x4(__fmul_rn(y[0], inv[0]), __fmul_rn(y[1], inv[1]), __fmul_rn(y[2], inv[2]),
                                          __fmul_rn(y[3], inv[3])),
                                     i8x4(__fmul_rn(y[4], inv[4]), __fmul_rn(y[5], inv[5]), __fmul_rn(y[6], inv[6]),
                                          __fmul_rn(y[7], inv[7])));
          *reinterpret_cast<uint2*>(dst + (base + tok) * kDPad + 8 * u) = w;
          continue;
        }
        const uint2 w = make_uint2(e4m3x4(__fmul_rn(y[0], inv[0]), __fmul_rn(y[1], inv[1]), __fmul_rn(y[2], inv[2]),
                                          __fmul_rn(y[3], inv[3])),
                                   e4m3x4(__fmul_rn(y[4], inv[4]), __fmul_rn(y[5], inv[5]), __fmul_rn(y[6], inv[6]),
                                          __fmul_rn(y[7], inv[7])));
        *reinterpret_cast<uint2*>(dst + (base + tok) * kDPad + 8 * u) = w;
      }
    }
  }
}

}  // namespace

cudaError_t launch_fp8_quant(const sla_shape& s, const void* q, const void* k, const void* v, const WsLayout& L,
                             char* ws, cudaStream_t st, bool int8_qk) {
  const int BH = s.B * s.H;
  const int nb128 = ceil_div(s.N, 128);
  float* mu = reinterpret_cast<float*>(ws + L.mu);
  float* vam = reinterpret_cast<float*>(ws + L.sv);
  fp8_stats_kernel<<<BH, 128, 0, st>>>(reinterpret_cast<const float*>(ws + L.kstat),
                                       reinterpret_cast<const float*>(ws + L.vstat), mu, vam, L.nsplit, s.N);
  dim3 grid(nb128, BH);
  auto* q8 = reinterpret_cast<uint8_t*>(ws + L.q8);
  auto* k8 = reinterpret_cast<uint8_t*>(ws + L.k8);
  auto* v8 = reinterpret_cast<uint8_t*>(ws + L.v8);
  auto* sq = reinterpret_cast<float*>(ws + L.sq);
  auto* sk = reinterpret_cast<float*>(ws + L.sk);
  auto run = [&](auto kernel, const auto* tq, const auto* tk, const auto* tv) {
    kernel<<<grid, 256, 0, st>>>(tq, tk, tv, mu, vam, q8, k8, v8, sq, sk, s.N, s.d, nb128);
  };
  using BF = __nv_bfloat16;
  if (s.in_dtype == SLA_BF16) {
    const auto* tq = static_cast<const BF*>(q);
    const auto* tk = static_cast<const BF*>(k);
    const auto* tv = static_cast<const BF*>(v);
    if (int8_qk) run(fp8_quant_kernel<BF, true>, tq, tk, tv);
    else run(fp8_quant_kernel<BF, false>, tq, tk, tv);
  } else {
    const auto* tq = static_cast<const float*>(q);
    const auto* tk = static_cast<const float*>(k);
    const auto* tv = static_cast<const float*>(v);
    if (int8_qk) run(fp8_quant_kernel<float, true>, tq, tk, tv);
    else run(fp8_quant_kernel<float, false>, tq, tk, tv);
  }
  return cudaGetLastError();
}

cudaError_t launch_prepare(const sla_shape& s, const void* k, const void* v, int phi, const WsLayout& L,
                           char* ws, cudaStream_t st) {
  const int BH = s.B * s.H;
  const int nkv = ceil_div(s.N, s.bkv);
  __half* phik = reinterpret_cast<__half*>(ws + L.phik);
  __half* v16 = reinterpret_cast<__half*>(ws + L.v16);
  __nv_bfloat16* khat = L.need_hat ? reinterpret_cast<__nv_bfloat16*>(ws + L.khat) : nullptr;
  float* hpart = reinterpret_cast<float*>(ws + L.hpart);
  float* zpart = reinterpret_cast<float*>(ws + L.zpart);
  int* status = reinterpret_cast<int*>(ws + L.status);
  dim3 grid(L.nsplit, BH);
  cudaError_t e;
  if (s.in_dtype == SLA_BF16 && s.d == kDPad) {
    CUtensorMap mk, mv, mpo, mvo;
    if ((e = encode_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, s.N, BH, 64)) != cudaSuccess) return e;
    if ((e = encode_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, s.N, BH, 64)) != cudaSuccess) return e;
    if ((e = encode_map(&mpo, phik, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, s.N, BH, 64)) != cudaSuccess) return e;
    if ((e = encode_map(&mvo, v16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, s.N, BH, 64)) != cudaSuccess) return e;
    e = cudaFuncSetAttribute(lin_prepass_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTPreSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(lin_prepass_tma_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    lin_prepass_tma_kernel<<<grid, kPreThreads, kTPreSmem, st>>>(
        mk, mv, mpo, mvo, hpart, zpart, reinterpret_cast<float*>(ws + L.zblk), reinterpret_cast<float*>(ws + L.kstat),
        reinterpret_cast<float*>(ws + L.vstat), reinterpret_cast<float*>(ws + L.kbar), s.N, nkv, L.nsplit, phi,
        status);
  } else if (s.in_dtype == SLA_BF16) {
    e = cudaFuncSetAttribute(lin_prepass_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kPreSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(lin_prepass_kernel<__nv_bfloat16>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               100);
    if (e != cudaSuccess) return e;
    lin_prepass_kernel<__nv_bfloat16><<<grid, kPreThreads, kPreSmem, st>>>(
        static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), phik, v16, khat, hpart,
        zpart, reinterpret_cast<float*>(ws + L.zblk), reinterpret_cast<float*>(ws + L.kstat),
        reinterpret_cast<float*>(ws + L.vstat), s.N, s.d, nkv, L.nsplit, phi, status);
  } else {
    e = cudaFuncSetAttribute(lin_prepass_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPreSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(lin_prepass_kernel<float>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    lin_prepass_kernel<float><<<grid, kPreThreads, kPreSmem, st>>>(
        static_cast<const float*>(k), static_cast<const float*>(v), phik, v16, khat, hpart, zpart,
        reinterpret_cast<float*>(ws + L.zblk), reinterpret_cast<float*>(ws + L.kstat),
        reinterpret_cast<float*>(ws + L.vstat), s.N, s.d, nkv, L.nsplit, phi, status);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  float* sig = reinterpret_cast<float*>(ws + L.sigma);
  zsum_kernel<<<BH, 128, 0, st>>>(zpart, reinterpret_cast<float*>(ws + L.ztot), sig, L.nsplit);
  const long long n = static_cast<long long>(BH) * kDPad * kDPad;
  hsum_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(hpart, sig,
                                                                      reinterpret_cast<__half*>(ws + L.hs16), BH,
                                                                      L.nsplit);
  return cudaGetLastError();
}

cudaError_t launch_qhat(const sla_shape& s, const void* q, const WsLayout& L, char* ws, cudaStream_t st) {
  const long long rows = static_cast<long long>(s.B) * s.H * s.N;
  __nv_bfloat16* qhat = reinterpret_cast<__nv_bfloat16*>(ws + L.qhat);
  const unsigned blocks = static_cast<unsigned>((rows * 16 + 255) / 256);
  if (s.in_dtype == SLA_BF16)
    qhat_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q), qhat, rows, s.d);
  else
    qhat_kernel<float><<<blocks, 256, 0, st>>>(static_cast<const float*>(q), qhat, rows, s.d);
  return cudaGetLastError();
}

}  // namespace sla
