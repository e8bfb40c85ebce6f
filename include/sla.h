/*
 * sla.h -- C ABI of libsla: SLA2 / SLA sparse-linear attention forward on
 * NVIDIA B200 (sm_100a).
 *
 * The pages this follows:
 *   [SLA2-deep] "SLA2 深度解读：97% 稀疏、18.7 倍注意力加速，它和 DeepSeek DSA 的可学习
 *               Indexer 到底差在哪" (jefxiong.cn), sections 04 (formulation),
 *               05 (learnable router), 07 (QAT), 08 (inference kernel).
 *   [SLA2-sum]  "SLA2: Sparse-Linear Attention with Learnable Routing and QAT"
 *               (gist.science), section 2 "Methodology: SLA2".
 *   [SLA]       "SLA: Beyond Sparsity in Diffusion Transformers via
 *               Fine-Tunable Sparse-Linear Attention" (papernotes.org),
 *               关键设计 2 (compressed map, three labels), 3 (linear branch,
 *               O = O_s + Proj(O_l)), 4 (fused kernel).
 *
 * Conventions for every entry point
 *   - Q, K, V are contiguous [B, H, N, d] (row-major, d fastest) in device
 *     memory, dtype SLA_BF16 or SLA_F32, base addresses 16-byte aligned.
 *     Query block i holds tokens [i*bq, min((i+1)*bq, N)); key block j holds
 *     [j*bkv, min((j+1)*bkv, N)); tokens past N do not exist (ragged last
 *     blocks are masked, never padded).
 *   - Ownership: the caller allocates and owns every buffer (inputs, outputs
 *     and the workspace `ws`).  The library allocates nothing, frees nothing,
 *     keeps no state between calls and does not synchronise the stream
 *     (except sla_read_device_status).  Every call only enqueues kernels on
 *     `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Errors: invalid arguments are reported before anything is launched
 *     (SLA_ERR_INVALID_ARG, SLA_ERR_UNSUPPORTED, SLA_ERR_ALIGNMENT,
 *     SLA_ERR_WORKSPACE).  A failed launch returns SLA_ERR_CUDA.  Errors found
 *     on the device (a bounded wait that ran out, an out-of-range block index)
 *     are written to a status word in `ws` and read with
 *     sla_read_device_status.  No call traps, asserts or hangs the device.
 *   - Supported: 8 <= d <= 128 with d % 8 == 0; bq in {64, 128}; bkv == 64;
 *     1 <= N <= 131072; B*H >= 1.
 */
#ifndef SLA_H_
#define SLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SLA_OK = 0,
  SLA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad enum value */
  SLA_ERR_UNSUPPORTED = 2,   /* valid but outside the supported set above */
  SLA_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned */
  SLA_ERR_WORKSPACE = 4,     /* ws too small (see sla_workspace_size) */
  SLA_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
  SLA_ERR_TIMEOUT = 6,       /* device: a bounded wait ran out */
  SLA_ERR_DEVICE_INDEX = 7   /* device: a block index out of [0, n_kv) */
} sla_status;

typedef enum { SLA_F32 = 0, SLA_BF16 = 1 } sla_dtype;

/* Linear-attention feature map phi [SLA 损失函数/训练策略, 关键设计 3]:
 * ELU(x)+1, or a softmax over the d channels of each token. */
typedef enum { SLA_PHI_ELU1 = 0, SLA_PHI_SOFTMAX = 1 } sla_phi;

/* Router output kind: SLA2 hard top-k [SLA2-deep §05], or SLA's three labels
 * critical / marginal / negligible [SLA 关键设计 2]. */
typedef enum { SLA_MODE_SLA2_TOPK = 0, SLA_MODE_SLA_3WAY = 1 } sla_route_mode;

/* OR into sla_route's mode: take the key-block means from ws, where
 * sla_prepare wrote them while it streamed K (bf16 inputs with d = 128 only),
 * instead of reading K again.  Same arithmetic, so the same bits; sla_prepare
 * must have run on these K and this ws, earlier on the same stream. */
#define SLA_ROUTE_KBAR_FROM_WS 0x10

/* flags for the attention entry points */
#define SLA_FLAG_PREPARED 1u  /* ws already holds sla_prepare's results for these K, V */
#define SLA_FLAG_FP8 2u       /* low-bit (e4m3) sparse branch [SLA2-deep §07], SLA2 only */
/* The page's other low-bit format ("INT8 or FP8" [SLA2-deep §07]): Q and
 * K - mean(K) as INT8 codes rint(x * 127 / amax) (ties to even, saturated to
 * +-127, one scale amax / 127 per 128-token block), S as an exact integer
 * product; P and V in e4m3 as with SLA_FLAG_FP8.  SLA2 only; excludes
 * SLA_FLAG_FP8; the workspace is sized with SLA_WS_FP8. */
#define SLA_FLAG_INT8 4u
/* Test hook for the device-side failure detection, not for production use:
 * every bounded wait of the attention kernel gives up as soon as it is not
 * already satisfied (limit 0 instead of 1 s), as a wait that ran out would.
 * The kernel then stops issuing work, drains the copies and tensor-core
 * products it started, frees its tensor memory and returns; the call's output
 * is undefined and sla_read_device_status reports SLA_ERR_TIMEOUT.  No wait
 * is left unsatisfied on purpose: the limit, not a missing arrival, ends it. */
#define SLA_FLAG_WAIT_TEST 8u

/* OR into the mode of sla_workspace_size to include the buffers of the
 * low-bit sparse branch (e4m3 copies of Q, K - mean(K), V and their scales). */
#define SLA_WS_FP8 0x100

typedef struct {
  int B, H, N, d;   /* batch, heads, tokens, head dim */
  int bq, bkv;      /* query / key block sizes (tokens) */
  int in_dtype;     /* sla_dtype of Q, K, V */
} sla_shape;

/* Human-readable name of a status code (static storage). */
const char* sla_status_string(sla_status s);

/* One line on the last host-side failure of this thread (which argument was
 * rejected, or which CUDA call failed and why); "" if none yet. */
const char* sla_last_error_detail(void);

/* Blocks kept per query block for a keep fraction "k%" [SLA2-deep §05]:
 * round-half-up(ratio * n_kv), at least 1 when ratio > 0, clamped to
 * [0, n_kv].  (The pages give only the percentage.) */
int sla_keep_count(double ratio, int n_kv);

/* Bytes of device workspace the calls below need for this shape and mode
 * (optionally | SLA_WS_FP8).  Returns 0 for an invalid shape.  One workspace serves sla_route,
 * sla_prepare and the attention calls; calls that share it must be ordered
 * on one stream. */
size_t sla_workspace_size(const sla_shape* shape, int mode);

/* Zero the workspace's device status word (enqueued on stream).  Call once
 * after allocating ws (a zero-filled allocation also works). */
sla_status sla_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Router [SLA2-deep §05; SLA 关键设计 2; SLA2-sum §2.B]:
 *   Qbar = pool_bq(Q), Kbar = pool_bkv(K)          (block means, valid tokens)
 *   Qt = Qbar Wq, Kt = Kbar Wk                     (Wq, Wk: d x d row-major fp32,
 *                                                   16-byte aligned, shared by
 *                                                   all heads; NULL = identity
 *                                                   = SLA heuristic)
 *   s[i,j] = Qt_i . Kt_j
 * then per query block i, with key blocks ordered by (s desc, index asc):
 *   SLA2: the first k_keep are kept;
 *   SLA : the first k_keep are critical (+1), the last k_neg negligible (-1).
 * All of this is fixed-order fp32 (sums in ascending index order from +0.0;
 * the means by one division; the projections and scores as chains of
 * multiply-adds, each rounded once), so the selection is reproducible bit
 * for bit.  The 1/sqrt(d) and softmax of SLA's
 * compressed map are not applied: both are monotone per row.
 * Outputs (device):
 *   kept_idx   int32 [B,H,n_q,k_keep], ascending per row (k_keep may be 0)
 *   labels     int8  [B,H,n_q,n_kv] (nullable): SLA2 1/0; SLA +1/0/-1
 *   scores_dbg fp32  [B,H,n_q,n_kv] (nullable): the raw scores s
 * Requires n_kv <= 2048 and k_keep + k_neg <= n_kv (k_neg = 0 for SLA2).
 * mode may carry SLA_ROUTE_KBAR_FROM_WS (bf16, d = 128; else UNSUPPORTED). */
sla_status sla_route(const sla_shape* shape, const void* q, const void* k,
                     const float* Wq, const float* Wk, int mode, int k_keep,
                     int k_neg, int32_t* kept_idx, int8_t* labels,
                     float* scores_dbg, void* ws, size_t ws_bytes,
                     void* stream);

/* SoftTop-k router mask, the differentiable stand-in for the hard Top-k while
 * the router is trained [SLA2-deep §06, Stage 1]:
 *   M[i,j] = sigmoid(s[i,j] / tau + lambda_i)
 * with s the router scores exactly as sla_route computes them (same kernels,
 * same bits) and lambda_i found by bisection so that sum_j M[i,j] = k_keep
 * (the row's budget; the pages use tau = 0.1).  fp32: x = s / tau, the
 * bracket [-max(x) - 40, -min(x) + 40], halved until its midpoint no longer
 * moves; k_keep == 0 gives M = 0 (lambda = -inf), k_keep == n_kv gives M = 1
 * (lambda = +inf).
 * Outputs (device, caller-owned):
 *   mask   fp32 [B,H,n_q,n_kv]
 *   lambda fp32 [B,H,n_q] (nullable)
 * tau must be positive and finite; 0 <= k_keep <= n_kv <= 2048.  Same
 * workspace and argument rules as sla_route. */
sla_status sla_route_soft(const sla_shape* shape, const void* q, const void* k,
                          const float* Wq, const float* Wk, int k_keep, float tau,
                          float* mask, float* lambda, void* ws, size_t ws_bytes,
                          void* stream);

/* Router without a workspace.  The pages have no counterpart to this entry
 * point: it exists for callers that cannot give the library device memory,
 * for example code that runs under another framework's memory manager and
 * may not allocate outside it, or that must not call cudaMalloc where it
 * routes.  It computes exactly what sla_route computes (same kernels, same
 * bit-exact results) with the same arguments minus ws / ws_bytes, except that
 * mode may not carry SLA_ROUTE_KBAR_FROM_WS (there is no workspace holding
 * the prepass's key-block means: SLA_ERR_INVALID_ARG).  Its scratch is a
 * 16 MiB array compiled into the library, held by every GPU that loads
 * libsla until the process exits.
 *   - Shapes whose scratch, B*H*(n_q + n_kv)*d floats (the projected block
 *     means of Q and K, each piece rounded up to 256 bytes), exceeds 16 MiB
 *     are rejected with SLA_ERR_WORKSPACE before any launch
 *     (sla_last_error_detail says how much was needed).  The 1.3B-shape
 *     workload needs 4.7 MB.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  The address is kept with the id of the
 *     CUDA context it belongs to; a call that finds another context current
 *     (after cudaDeviceReset, say) looks it up again, so that call too should
 *     come before any capture.
 *   - All calls share the array: calls that overlap on the GPU race.  Nothing
 *     in it needs to start at zero: each call writes every value that reaches
 *     its results before reading it.
 *   - Every rejected argument also sets sla_last_error_detail.
 *   - Nothing is allocated or freed. */
sla_status sla_route_noalloc(const sla_shape* shape, const void* q, const void* k,
                             const float* Wq, const float* Wk, int mode, int k_keep,
                             int k_neg, int32_t* kept_idx, int8_t* labels,
                             float* scores_dbg, void* stream);

/* Linear-branch totals [SLA 关键设计 3, 4; SLA2-deep §08]: per (b,h)
 *   H_tot = sum_n phi(k_n)^T v_n  (d x d),  Z_tot = sum_n phi(k_n)  (d)
 * over all N tokens, plus the per-token phi(K) and V staged in ws for the
 * attention kernel.  The attention calls run this themselves unless
 * SLA_FLAG_PREPARED is passed.  K, V as in the conventions. */
sla_status sla_prepare(const sla_shape* shape, const void* k, const void* v,
                       int phi, void* ws, size_t ws_bytes, void* stream);

/* SLA2 attention forward [SLA2-deep §04, §08; SLA2-sum §2.A]:
 *   O_s = softmax over the kept key blocks of Q K^T / sqrt(d), times V
 *   O_l = phi(Q) H_i / (phi(Q) Z_i),  H_i, Z_i over the key blocks not kept
 *   O   = alpha_i * O_s + (1 - alpha_i) * O_l
 * kept_idx: int32 [B,H,n_q,k_keep], ascending per row, values in [0, n_kv)
 *   (as written by sla_route).  k_keep == 0 -> O_s = 0; k_keep == n_kv ->
 *   O_l = 0.
 * alpha: fp32 [B,H,n_q], one mixing ratio per query block, already in [0,1].
 * out: [B,H,N,d] of out_dtype (SLA_F32 or SLA_BF16), fully overwritten.
 * flags: SLA_FLAG_PREPARED to skip the sla_prepare step. */
sla_status sla2_attn_fwd(const sla_shape* shape, const void* q, const void* k,
                         const void* v, const int32_t* kept_idx, int k_keep,
                         const float* alpha, int phi, unsigned flags,
                         void* out, int out_dtype, void* ws, size_t ws_bytes,
                         void* stream);

/* SLA attention forward [SLA 关键设计 2, 3, 4]:
 *   O_s = softmax attention over the critical blocks (label +1)
 *   O_l = linear attention over the marginal blocks (label 0); negligible
 *         blocks (label -1) are skipped
 *   O   = O_s + O_l W_proj,  W_proj bf16 [d_in][d_out] row-major, no bias
 * labels: int8 [B,H,n_q,n_kv] with values in {-1, 0, 1} (any counts per row).
 * ws must be sized with mode SLA_MODE_SLA_3WAY.  Other arguments as above. */
sla_status sla_attn_fwd(const sla_shape* shape, const void* q, const void* k,
                        const void* v, const int8_t* labels, const void* Wproj,
                        int phi, unsigned flags, void* out, int out_dtype,
                        void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace sla2_attn_bwd needs for this shape (0 for an
 * invalid shape).  CUDA-core path: the status word, H_tot, Z_tot and their
 * gradients per (b,h), and a [B,H,N,128] fp32 buffer of key-side sums.
 * Tensor-core path (bf16, d = 128, bq = 128): the forward's SLA2 workspace
 * (sla_workspace_size with SLA_MODE_SLA2_TOPK) followed by the per-row
 * statistics, fp16 phi(Q), the inverse block lists, the per-tile dH (fp16)
 * and dZ partials, dH_tot, dZ_tot and a scaled fp16 copy of dH_tot. */
size_t sla2_attn_bwd_workspace_size(const sla_shape* shape);

/* Gradients of the SLA2 forward [SLA 关键设计 4; SLA2-deep §07; SLA2-sum §2.C]
 * for the upstream gradient dout, with the block mask held fixed (the hard
 * Top-k passes no gradient):
 *   dO_s = alpha dO, dO_l = (1 - alpha) dO, dalpha_i = sum over the rows of
 *   query block i of dO . (O_s - O_l); the sparse branch back-propagated as
 *   FlashAttention does, the linear branch through dH_i, dZ_i formed from the
 *   totals minus the kept blocks' share.
 * The gradients are taken on the original (unquantised) inputs, so this is
 *   also the backward of the e4m3 forward (SLA_FLAG_FP8): the low-bit
 *   quantisation is forward-only [SLA2-deep §07].
 * Inputs q, k, v, kept_idx, k_keep, alpha, phi as for sla2_attn_fwd (kept
 * indices distinct per row); dout [B,H,N,d] of the input dtype.
 * Outputs (fp32, caller-owned, fully overwritten): dq, dk, dv [B,H,N,d],
 *   dalpha [B,H,n_q].
 * Two paths: bf16 inputs with d = 128 and bq = 128 run on the tensor cores
 *   (bf16 / fp16 operands, fp32 accumulation; every output written once in a
 *   fixed order, so runs agree bit for bit; errors about 2e-3 of each tensor's
 *   largest entry); every other shape runs in fp32 on the CUDA cores, where dk,
 *   dv and dalpha are accumulated with atomic adds after a zero fill, so their
 *   last bits can differ between runs.
 * ws: its own workspace of sla2_attn_bwd_workspace_size bytes, 256-byte
 *   aligned, status word zeroed once (sla_workspace_init); the call zeroes
 *   the rest itself.  Out-of-range block indices are skipped and reported in
 *   the status word (sla_read_device_status). */
sla_status sla2_attn_bwd(const sla_shape* shape, const void* q, const void* k,
                         const void* v, const int32_t* kept_idx, int k_keep,
                         const float* alpha, int phi, const void* dout,
                         float* dq, float* dk, float* dv, float* dalpha,
                         void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace sla_attn_bwd needs for this shape (0 for an
 * invalid shape): sla2_attn_bwd's, plus the critical / negligible block lists,
 * a [B,H,N,128] fp32 buffer of the O_l rows and the dW_proj partial sums. */
size_t sla_attn_bwd_workspace_size(const sla_shape* shape);

/* Gradients of the SLA forward [SLA 关键设计 4] for the upstream gradient
 * dout, with the labels held fixed:
 *   dO_s = dO, dO_l = dO W_proj^T, dW_proj = sum over the rows of every head
 *   of O_l^T dO (W_proj is shared by the heads); the critical blocks take the
 *   sparse branch back-propagated as FlashAttention does, the marginal blocks
 *   the linear branch through dH_i, dZ_i (the totals minus the critical and
 *   negligible blocks' share), the negligible blocks get nothing.
 * Inputs q, k, v, labels, Wproj, phi as for sla_attn_fwd; dout [B,H,N,d] of
 *   the input dtype.
 * Outputs (fp32, caller-owned, fully overwritten): dq, dk, dv [B,H,N,d],
 *   dWproj [d][d] (d_in x d_out, as Wproj).  dk and dv are accumulated with
 *   atomic adds after a zero fill, so their last bits can differ between runs;
 *   dWproj is summed in a fixed order.
 * ws: its own workspace of sla_attn_bwd_workspace_size bytes, 256-byte
 *   aligned, status word zeroed once (sla_workspace_init).  A label outside
 *   {-1, 0, 1} is reported in the status word (sla_read_device_status) and
 *   the block is treated as marginal. */
sla_status sla_attn_bwd(const sla_shape* shape, const void* q, const void* k,
                        const void* v, const int8_t* labels, const void* Wproj,
                        int phi, const void* dout, float* dq, float* dk,
                        float* dv, float* dWproj, void* ws, size_t ws_bytes,
                        void* stream);

/* Bytes of device memory sla2_forward_host needs (0 for invalid arguments):
 * the workspace of sla_workspace_size (with SLA_WS_FP8 when flags carry
 * SLA_FLAG_FP8 or SLA_FLAG_INT8) followed by device copies of Q, K, V, Wq, Wk, alpha, the kept
 * lists and the output, each 256-byte aligned. */
size_t sla2_forward_host_device_bytes(const sla_shape* shape, int k_keep, int out_dtype, unsigned flags);

/* One whole SLA2 forward from host memory [SLA2-deep §04, §05, §08]: the
 * router (top-k_keep per query block), the linear-branch totals and the
 * attention call, exactly as sla_route + sla_prepare + sla2_attn_fwd compute
 * them, with the inputs copied in and the output copied out on `stream`.
 *   q, k, v  host [B,H,N,d] of shape->in_dtype;  Wq, Wk host d x d fp32
 *            (nullable = identity);  alpha host fp32 [B,H,n_q];
 *   out      host [B,H,N,d] of out_dtype (SLA_F32 / SLA_BF16);
 *   kept_out host int32 [B,H,n_q,k_keep] (nullable): the router's kept lists.
 *   flags    0, SLA_FLAG_FP8 or SLA_FLAG_INT8 (the low-bit sparse branches).
 *   dev      device memory of sla2_forward_host_device_bytes bytes, 256-byte
 *            aligned, caller-owned; its first 256 bytes are the workspace
 *            status word (zero it once with sla_workspace_init, read it with
 *            sla_read_device_status(dev, stream)).
 * Everything is enqueued on `stream`; the call returns without waiting, so
 * the host buffers must stay valid (and out unread) until the stream is
 * synchronised.  Page-locked host memory lets the copies run asynchronously;
 * one cudaMemcpyAsync is issued per buffer.  Same argument rules as the calls
 * it combines. */
sla_status sla2_forward_host(const sla_shape* shape, const void* q, const void* k,
                             const void* v, const float* Wq, const float* Wk,
                             const float* alpha, int k_keep, int phi, unsigned flags,
                             void* out, int out_dtype, int32_t* kept_out, void* dev,
                             size_t dev_bytes, void* stream);

/* Synchronise `stream`, then return (and clear) the device status word that
 * kernels write when a bounded wait runs out or a block index is out of
 * range.  SLA_OK when no device error happened. */
sla_status sla_read_device_status(void* ws, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SLA_H_ */
