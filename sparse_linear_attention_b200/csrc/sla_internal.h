// sla_internal.h -- definitions shared by the libsla host code and kernels.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/sla.h"

namespace sla {

constexpr int kDPad = 128;        // head dim as stored for the tensor-core path
constexpr int kBlockKV = 64;      // key block size (tokens)
constexpr int kMaxNKV = 2048;     // router limit on key blocks per head
constexpr int kMaxN = 131072;     // token limit (n_kv <= 2048 at bkv = 64)
constexpr int kNumSMs = 148;

// Every wait in the kernels gives up after this long and reports
// SLA_ERR_TIMEOUT instead of hanging the GPU.
constexpr unsigned long long kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

// Device workspace layout.  All offsets are 256-byte aligned.
struct WsLayout {
  size_t status = 0;  // int32 status word (+ padding)
  size_t qt = 0, kt = 0;      // fp32 [d][rows] per head: projected block means of Q, K (K rows kt_stride long)
  size_t phik = 0;            // fp16 [BH, N, 128]  phi(K), zero past d
  size_t v16 = 0;             // fp16 [BH, N, 128]  V, zero past d
  size_t qhat = 0, khat = 0;  // bf16 [BH, N, 128]  Q, K (only when need_hat)
  size_t hpart = 0, zpart = 0;  // fp32 [BH, nsplit, 128, 128], [BH, nsplit, 128]
  size_t hs16 = 0, ztot = 0;    // fp16 [BH, 128, 128] = H_tot / sigma, fp32 [BH, 128] = Z_tot
  size_t sigma = 0;             // fp32 [BH]: per-head power of two >= max_e Z_tot[e]
  size_t zblk = 0;              // fp32 [BH, n_kv, 128]: colsum of phi(K) per key block
  size_t kbar = 0;              // fp32 [BH, n_kv, 128]: key-block means for the router (bf16, d = 128 prepass)
  size_t kstat = 0, vstat = 0;  // fp32 [BH, nsplit, 128]: per-split column sum of K, column absmax of V
  // low-bit sparse branch (only with SLA_WS_FP8)
  size_t q8 = 0, k8 = 0, v8 = 0;  // e4m3 [BH, N, 128]: Q, K - mean(K), V
  size_t sq = 0, sk = 0;          // fp32 [BH, ceil(N/128)]: per-block scales of Q and K - mean(K)
  size_t mu = 0, sv = 0;          // fp32 [BH, 128]: column mean of K, column absmax of V
  bool fp8 = false;
  size_t lists = 0;             // SLA: int32 [BH, n_q, 2, n_kv] critical / negligible lists
  size_t counts = 0;            // SLA: int32 [BH, n_q, 2]
  size_t total = 0;
  int nsplit = 1;
  bool need_hat = false;
};

// Workspace of the backward (sla2_attn_bwd): status word first, as in WsLayout.
struct BwdLayout {
  size_t status = 0;
  size_t htot = 0, ztot = 0;    // fp32 [BH, 128, 128], [BH, 128]: H_tot, Z_tot
  size_t dhtot = 0, dztot = 0;  // fp32 [BH, 128, 128], [BH, 128]: their gradients
  size_t dphik = 0;             // fp32 [BH, N, 128]: kept blocks' share of dL/dphi(K)
  size_t lists = 0, counts = 0;  // SLA: int32 [BH, n_q, 2, n_kv] critical / negligible lists, [BH, n_q, 2] counts
  size_t ol = 0;                // SLA: fp32 [BH, N, 128]: O_l rows for dW_proj
  size_t wpart = 0;             // SLA: fp32 [splits, 128, 128]: dW_proj partial sums
  size_t total = 0;
};

// Record the one-line detail that sla_last_error_detail() returns.
void set_error_detail(const char* msg);

// Workspace of the tensor-core backward (bf16, d = 128, b_q = 128): the
// forward's workspace first (its status word at offset 0), then the per-row
// statistics, phi(Q), the inverse block lists and the reduction buffers.
struct BwdTcLayout {
  WsLayout fwd;
  size_t rows = 0;            // fp32 [BH * N, 8]: lse2, D, s, dden, dalpha share
  size_t phiq = 0;            // fp16 [BH, N, 128]
  size_t inv = 0, inv_n = 0;  // int32 [BH, n_kv, n_q], [BH, n_kv]
  size_t dhpart = 0, dzpart = 0;  // fp16 [BH * n_q, 128, 128] = -sigma dH_i, fp32 [BH * n_q, 128] = dZ_i
  size_t dhtot = 0, dztot = 0;    // fp32 [BH, 128, 128], [BH, 128]
  size_t dh16 = 0, tau = 0;   // fp16 [BH, 128, 128] = tau dH_tot; fp32 [BH] power-of-two scale tau
  size_t total = 0;
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Row stride (floats) of the projected key means: n_kv rounded up to 4, so
// every row starts on 16 bytes for the score kernel's async copies.
inline int kt_stride(int nkv) { return (nkv + 3) & ~3; }

inline WsLayout ws_layout(const sla_shape& s, int mode_flags) {
  const int mode = mode_flags & 0xFF;
  WsLayout L;
  L.fp8 = (mode_flags & SLA_WS_FP8) != 0;
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  const int nq = ceil_div(s.N, s.bq), nkv = ceil_div(s.N, s.bkv);
  L.need_hat = (s.d != kDPad) || (s.in_dtype == SLA_F32);
  // prepass splits per head: one wave of two CTAs per SM (rounding up would leave a
  // few CTAs for a second wave and double the prepass time)
  int ns = (2 * kNumSMs) / static_cast<int>(BH > 0 ? BH : 1);
  L.nsplit = ns < 1 ? 1 : (ns > nkv ? nkv : ns);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.status = take(256);
  L.qt = take(BH * nq * s.d * 4);
  L.kt = take(BH * static_cast<size_t>(kt_stride(nkv)) * s.d * 4);
  L.phik = take(BH * s.N * kDPad * 2);
  L.v16 = take(BH * s.N * kDPad * 2);
  if (L.need_hat) {
    L.qhat = take(BH * s.N * kDPad * 2);
    L.khat = take(BH * s.N * kDPad * 2);
  }
  L.hpart = take(BH * L.nsplit * kDPad * kDPad * 4);
  L.zpart = take(BH * L.nsplit * kDPad * 4);
  L.hs16 = take(BH * kDPad * kDPad * 2);
  L.ztot = take(BH * kDPad * 4);
  L.sigma = take(BH * 4);
  L.zblk = take(BH * static_cast<size_t>(nkv) * kDPad * 4);
  L.kbar = take(BH * static_cast<size_t>(nkv) * kDPad * 4);
  L.kstat = take(BH * L.nsplit * kDPad * 4);
  L.vstat = take(BH * L.nsplit * kDPad * 4);
  if (L.fp8) {
    const size_t nb128 = static_cast<size_t>(ceil_div(s.N, 128));
    L.q8 = take(BH * s.N * kDPad);
    L.k8 = take(BH * s.N * kDPad);
    L.v8 = take(BH * s.N * kDPad);
    L.sq = take(BH * nb128 * 4);
    L.sk = take(BH * nb128 * 4);
    L.mu = take(BH * kDPad * 4);
    L.sv = take(BH * kDPad * 4);
  }
  if (mode == SLA_MODE_SLA_3WAY) {
    L.lists = take(BH * nq * 2 * static_cast<size_t>(nkv) * 4);
    L.counts = take(BH * nq * 2 * 4);
  }
  L.total = off;
  return L;
}

}  // namespace sla
