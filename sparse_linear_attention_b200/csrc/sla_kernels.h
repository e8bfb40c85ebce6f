// sla_kernels.h -- host-side launchers of the libsla kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "sla_internal.h"

namespace sla {

// Hard routing (kept_idx / labels) or, when soft_mask is non-null, the SoftTop-k
// mask and lambda with temperature tau.  kbar (nullable): the key-block means
// sla_prepare wrote, used instead of pooling K again.
cudaError_t launch_route(const sla_shape& s, const void* q, const void* k, const float* Wq, const float* Wk,
                         int mode, int k_keep, int k_neg, int32_t* kept_idx, int8_t* labels,
                         float* scores_dbg, const WsLayout& L, char* ws, cudaStream_t st, float tau = 0.0f,
                         float* soft_mask = nullptr, float* soft_lambda = nullptr, const float* kbar = nullptr);

BwdLayout bwd_layout(const sla_shape& s, bool sla_mode);

// Gradients of the SLA2 forward (backward.cu): zeroes dk, dv, dalpha and the
// workspace sums, then runs the three backward kernels on st.
cudaError_t launch_backward(const sla_shape& s, const void* q, const void* k, const void* v, const void* dout,
                            const int32_t* kept, int k_keep, const float* alpha, int phi, float* dq, float* dk,
                            float* dv, float* dalpha, char* ws, cudaStream_t st);

// The tensor-core SLA2 backward (backward_tc.cu) for bf16 inputs, d = 128,
// b_q = 128: same arguments as launch_backward, its own workspace layout.
BwdTcLayout bwd_tc_layout(const sla_shape& s);
bool bwd_tc_eligible(const sla_shape& s);
cudaError_t launch_backward_tc(const sla_shape& s, const void* q, const void* k, const void* v, const void* dout,
                               const int32_t* kept, int k_keep, const float* alpha, int phi, float* dq, float* dk,
                               float* dv, float* dalpha, char* ws, cudaStream_t st);

// Gradients of the SLA forward (backward.cu): the labels turned into lists,
// the same three kernels with the SLA weights, then the dW_proj reduction.
cudaError_t launch_sla_backward(const sla_shape& s, const void* q, const void* k, const void* v, const void* dout,
                                const int8_t* labels, const void* wproj, int phi, float* dq, float* dk, float* dv,
                                float* dwproj, char* ws, cudaStream_t st);

cudaError_t launch_prepare(const sla_shape& s, const void* k, const void* v, int phi, const WsLayout& L,
                           char* ws, cudaStream_t st);

// e4m3 copies of Q, K - mean(K), V and their scales (needs sla_prepare's statistics).
// 8-bit copies for the low-bit sparse branch: e4m3 Q, K - mean(K), V; with
// int8_qk the Q and K - mean(K) codes are INT8 instead (V stays e4m3).
cudaError_t launch_fp8_quant(const sla_shape& s, const void* q, const void* k, const void* v, const WsLayout& L,
                             char* ws, cudaStream_t st, bool int8_qk);

cudaError_t launch_qhat(const sla_shape& s, const void* q, const WsLayout& L, char* ws, cudaStream_t st);

cudaError_t launch_labels_to_lists(const sla_shape& s, const int8_t* labels, const WsLayout& L, char* ws,
                                   cudaStream_t st);
cudaError_t launch_labels_to_lists(const sla_shape& s, const int8_t* labels, int32_t* lists, int32_t* counts,
                                   int* status, cudaStream_t st);

struct SparseArgs {
  int BH, N, d, bq, nq, nkv;
  float sl2;                 // log2(e) / sqrt(d)
  const int32_t* crit_idx;   // per (bh, query block) row, list_stride apart: softmax blocks
  const int32_t* negl_idx;   // same rows: blocks that only leave the linear sum (SLA); nullable
  long long list_stride;     // elements between consecutive rows of both lists
  int crit_max, negl_max;    // list capacities
  const int32_t* counts;     // nullable: counts[2*row] = #crit, [2*row+1] = #negl; else crit_max, 0
  const float* alpha;        // SLA2: [BH, nq]; null for SLA
  const void* wproj;         // SLA: bf16 [d][d]; null for SLA2
  const float* sigma;        // [BH]: power of two >= max_e Z_tot[e]
  const float* ztot;         // [BH, 128]
  const float* zblk;         // [BH, nkv, 128]: per-block column sums of phi(K)
  void* out;
  int out_bf16;
  int tma_out;               // bf16 output, d = 128, bq = 128: 128-row tiles leave through a TMA store
  int phi;
  int* status;
  // low-bit sparse branch: 0 none (bf16), 1 e4m3 Q, K', P, V; 2 INT8 Q, K' with e4m3 P, V
  int fp8;
  int nb128;                 // ceil(N / 128)
  const float* sq;           // [BH, nb128] per-block scale of Q
  const float* sk;           // [BH, nb128] per-block scale of K - mean(K)
  const float* vamax;        // [BH, 128] column absmax of V
  const void* qsrc;          // bf16 [BH, N, 128] Q (for phi(Q) when the smem tile holds e4m3)
  unsigned long long wait_ns;  // limit of every bounded wait (the exit drains keep their own)
  // Backward statistics (SLA2, bf16 branch, d = 128; null otherwise): with the
  // upstream gradient bwd_do (bf16 [BH, N, 128]) the epilogue writes per row
  // bwd_rows[row * 8 + 0..4] = log2-sum-exp of the scaled kept scores,
  // D = alpha dO . O_s, s = (1 - alpha) / den, dden = -(1 - alpha) dO . O_l / den
  // and dO . (O_s - O_l).  out may then be null (no output written).
  const void* bwd_do;
  float* bwd_rows;
};

// 3-D tensor map over a [BH][N][128] 16-bit array: boxes of 64 channels x
// box_rows tokens, 128-byte swizzle, rows past N read as zero.
cudaError_t encode_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int N, int BH, int box_rows);
// Same over a [BH][N][128] byte array (e4m3), boxes of 128 bytes x box_rows.
cudaError_t encode_map8(CUtensorMap* map, const void* base, int N, int BH, int box_rows);

cudaError_t launch_sparse(const SparseArgs& a, const void* q_bf16_128, const void* k_bf16_128,
                          const void* phik16, const void* v16, const void* hs16, const void* q8, const void* k8,
                          const void* v8, cudaStream_t st);

}  // namespace sla
