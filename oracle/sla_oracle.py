"""CPU oracle for the SLA2 / SLA sparse-linear attention forward pass and its
gradients.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference leg may import this module.  The library
(sparse_linear_attention_b200) never imports it and shares no code with it.

Plain, slow and written to be checked by eye against the pages:

  [SLA2-sum]  "SLA2: Sparse-Linear Attention with Learnable Routing and QAT"
              (gist.science summary), section 2 "Methodology: SLA2".
  [SLA2-deep] "SLA2 深度解读：97% 稀疏、18.7 倍注意力加速，它和 DeepSeek DSA 的可学习
              Indexer 到底差在哪" (jefxiong.cn), sections 04 (formulation),
              05 (learnable router), 06 (two-stage training: SoftTop-k),
              07 (QAT), 08 (inference kernel).
  [SLA]       "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable
              Sparse-Linear Attention" (papernotes.org), 方法详解 / 关键设计 2
              (compressed map and three labels), 3 (linear branch and Proj),
              4 (fused kernel), 损失函数/训练策略 (phi, k_h, k_l, block sizes).

Precision.  Attention arithmetic is fp64 on the exact values of the input bytes.
The router is fixed-order fp32 (below) because a hard top-k must be reproduced
bit for bit; every fp32 step is one IEEE round-to-nearest-even operation:
  pooled mean : sum tokens in ascending order from +0.0, then divide by count;
  projection  : y[c] = fma(xbar[e], W[e,c], y[c]) for e ascending, from +0.0
                (each multiply-add rounded once);
  score       : s[i,j] = fma(qt[i,c], kt[j,c], s[i,j]) for c ascending, from +0.0.
Neither 1/sqrt(d) nor the softmax of the SLA compressed map is applied before
ranking: both are strictly increasing per row, so they cannot change a top-k.

Block conventions.  Query block i holds tokens [i*bq, min((i+1)*bq, N)), key
block j holds [j*bkv, min((j+1)*bkv, N)).  Tokens past N do not exist: they are
left out of every mean, softmax and sum.

Every function here has pins in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math

import numpy as np

F32 = np.float32
F64 = np.float64


# ----------------------------------------------------------------------------
# Router  [SLA2-deep §05], [SLA 关键设计 2], [SLA2-sum §2.B]
# ----------------------------------------------------------------------------

def keep_count(ratio: float, n_kv: int) -> int:
    """Blocks kept per row for a keep fraction "k%" [SLA2-deep §05]: the pages
    give only the percentage, so this reads it as round-half-up(ratio*n_kv),
    at least 1 when ratio > 0, clamped to [0, n_kv]."""
    if ratio <= 0.0:
        return 0
    k = int(math.floor(ratio * n_kv + 0.5))
    return max(1, min(n_kv, k))


def pool_blocks(x32: np.ndarray, b: int) -> np.ndarray:
    """Block mean-pooling pool(X) [SLA2-deep §05, SLA 关键设计 2].

    x32: float32 [B,H,N,d] -> float32 [B,H,ceil(N/b),d], fixed-order fp32.
    """
    x32 = np.asarray(x32, dtype=F32)
    B, H, N, d = x32.shape
    nb = -(-N // b)
    acc = np.zeros((B, H, nb, d), dtype=F32)
    counts = np.array([min((i + 1) * b, N) - i * b for i in range(nb)], dtype=np.int64)
    for t in range(b):
        live = np.nonzero(counts > t)[0]          # blocks that have a token at offset t
        rows = live * b + t
        acc[:, :, live, :] = acc[:, :, live, :] + x32[:, :, rows, :]
    return acc / counts.astype(F32)[None, None, :, None]


def fma32(a, b, c) -> np.ndarray:
    """fl32(a * b + c) with a single rounding, elementwise, for fp32 a, b, c.
    a * b is exact in fp64 (24 + 24 bits); the fp64 sum is then rounded to
    odd (when it is inexact, of the two fp64 neighbours of the exact value the
    one with an odd last bit), and rounding that to fp32 (53 >= 24 + 2 bits)
    gives the correctly rounded result (Boldo and Melquiond, rounding to odd)."""
    a = np.asarray(a, dtype=F32).astype(F64)
    b = np.asarray(b, dtype=F32).astype(F64)
    c = np.asarray(c, dtype=F32).astype(F64)
    p = a * b
    s = p + c
    bb = s - p
    e = (p - (s - bb)) + (c - bb)                 # exact error of the fp64 sum
    even = (np.asarray(s).view(np.uint64) & np.uint64(1)) == 0
    step = np.nextafter(s, np.where(e > 0, np.inf, -np.inf))
    s = np.where((e != 0) & even, step, s)
    return np.asarray(s, dtype=F64).astype(F32)


def project(xbar32: np.ndarray, w32) -> np.ndarray:
    """Learnable projection proj(X) = X W (no bias) [SLA2-deep §05]; W = None is
    the identity, which turns the router into SLA's pooled heuristic.  Each
    output is a chain of fused multiply-adds over e ascending from +0.0."""
    if w32 is None:
        return np.array(xbar32, dtype=F32, copy=True)
    xbar32 = np.asarray(xbar32, dtype=F32)
    w32 = np.asarray(w32, dtype=F32)
    d = xbar32.shape[-1]
    acc = np.zeros(xbar32.shape[:-1] + (w32.shape[1],), dtype=F32)
    for e in range(d):
        acc = fma32(xbar32[..., e:e + 1], w32[e, :], acc)
    return acc


def block_scores(qt32: np.ndarray, kt32: np.ndarray) -> np.ndarray:
    """Compressed score map P_c = proj_q(Qbar) proj_k(Kbar)^T [SLA2-deep §05],
    a chain of fused multiply-adds over c ascending from +0.0, without the
    monotone 1/sqrt(d) and softmax of [SLA 关键设计 2].
    qt32 [B,H,nq,d], kt32 [B,H,nkv,d] -> [B,H,nq,nkv]."""
    qt32 = np.asarray(qt32, dtype=F32)
    kt32 = np.asarray(kt32, dtype=F32)
    d = qt32.shape[-1]
    acc = np.zeros(qt32.shape[:-1] + (kt32.shape[-2],), dtype=F32)
    for c in range(d):
        acc = fma32(qt32[..., :, c, None], kt32[..., None, :, c], acc)
    return acc


def rank_order(scores: np.ndarray) -> np.ndarray:
    """Per row, key-block indices from best to worst: score descending, lower
    index first among equal scores (the pages do not say how ties break)."""
    return np.argsort(-scores, axis=-1, kind="stable")


def topk_blocks(scores: np.ndarray, k: int) -> np.ndarray:
    """Hard Top-k(k%, P_c) block mask as kept indices [SLA2-deep §05], ascending.
    Returns int32 [..., k]."""
    order = rank_order(scores)[..., :k]
    return np.sort(order, axis=-1).astype(np.int32)


def three_way_labels(scores: np.ndarray, k_h: int, k_l: int) -> np.ndarray:
    """SLA labels [SLA 关键设计 2]: top k_h blocks of each row critical (+1),
    bottom k_l negligible (-1), the rest marginal (0).  int8 [..., nkv]."""
    n_kv = scores.shape[-1]
    if k_h + k_l > n_kv:
        raise ValueError("k_h + k_l exceeds the number of key blocks")
    order = rank_order(scores)
    lab = np.zeros(scores.shape, dtype=np.int8)
    np.put_along_axis(lab, order[..., :k_h], np.int8(1), axis=-1)
    if k_l > 0:
        np.put_along_axis(lab, order[..., n_kv - k_l:], np.int8(-1), axis=-1)
    return lab


def sigmoid(z: np.ndarray) -> np.ndarray:
    """Logistic function 1 / (1 + e^-z) in fp64, written per sign so that
    neither branch overflows."""
    z = np.asarray(z, dtype=np.float64)
    out = np.empty_like(z)
    pos = z >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-z[pos]))
    ez = np.exp(z[~pos])
    out[~pos] = ez / (1.0 + ez)
    return out


def soft_topk(scores: np.ndarray, k: int, tau: float = 0.1, iters: int = 200):
    """SoftTop-k of the router map, the differentiable stand-in for the hard
    Top-k during the router's first training stage [SLA2-deep §06]:
    M[i, j] = sigmoid(P_c[i, j] / tau + lambda_i), with tau = 0.1 on the pages
    and lambda_i found by bisection so that each row's soft selections sum to
    the budget k.

    The row sum is strictly increasing in lambda, from 0 to n, so for
    0 < k < n the root is unique.  The bracket starts at
    [-max(s)/tau - 40, -min(s)/tau + 40], where the sum is below n * e^-40
    and above n - n * e^-40, and the interval is halved `iters` times (fp64).
    k <= 0 gives M = 0 (lambda = -inf), k >= n gives M = 1 (lambda = +inf).
    scores: [..., n]; returns (M float64 [..., n], lambda float64 [...])."""
    x = np.asarray(scores, dtype=np.float64) / tau
    n = x.shape[-1]
    lead = x.shape[:-1]
    if k <= 0:
        return np.zeros(x.shape), np.full(lead, -np.inf)
    if k >= n:
        return np.ones(x.shape), np.full(lead, np.inf)
    lo = -x.max(axis=-1) - 40.0
    hi = -x.min(axis=-1) + 40.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        f = sigmoid(x + mid[..., None]).sum(axis=-1)
        below = f < k
        lo = np.where(below, mid, lo)
        hi = np.where(below, hi, mid)
    lam = 0.5 * (lo + hi)
    return sigmoid(x + lam[..., None]), lam


def route(q, k, wq, wk, bq, bkv, mode="sla2", k_keep=0, k_neg=0):
    """Whole router: pool, project, score, select.  q, k: float32 views of the
    input bytes [B,H,N,d].  Returns (kept int32 [B,H,nq,k_keep] ascending,
    labels int8 [B,H,nq,nkv], scores float32 [B,H,nq,nkv]).  For mode "sla2"
    labels are 1 on kept blocks and 0 elsewhere; for "sla" kept lists the
    critical blocks."""
    qt = project(pool_blocks(q, bq), wq)
    kt = project(pool_blocks(k, bkv), wk)
    s = block_scores(qt, kt)
    if mode == "sla2":
        kept = topk_blocks(s, k_keep)
        lab = np.zeros(s.shape, dtype=np.int8)
        if k_keep > 0:
            np.put_along_axis(lab, kept.astype(np.int64), np.int8(1), axis=-1)
        return kept, lab, s
    lab = three_way_labels(s, k_keep, k_neg)
    kept = topk_blocks(s, k_keep)
    return kept, lab, s


# ----------------------------------------------------------------------------
# Feature map phi  [SLA 损失函数/训练策略, SLA 关键设计 3]
# ----------------------------------------------------------------------------

def phi(x: np.ndarray, kind: str = "elu1") -> np.ndarray:
    """Linear-attention feature map.  "elu1": ELU(x)+1 = x+1 for x>0, exp(x)
    otherwise.  "softmax": softmax over the channel axis of each token."""
    x = np.asarray(x, dtype=F64)
    if kind == "elu1":
        return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))
    if kind == "softmax":
        e = np.exp(x - x.max(axis=-1, keepdims=True))
        return e / e.sum(axis=-1, keepdims=True)
    raise ValueError(kind)


# ----------------------------------------------------------------------------
# Attention branches (fp64)
# ----------------------------------------------------------------------------

def _rows(i, b, N):
    return np.arange(i * b, min((i + 1) * b, N))


def _tokens_of(blocks, b, N):
    if len(blocks) == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([_rows(int(j), b, N) for j in blocks])


def sparse_branch(q, k, v, rows, keys):
    """O_s = P_s V with P_s the softmax of Q K^T/sqrt(d) over the selected keys
    only, i.e. P_1 renormalised per row [SLA2-deep §04, §08].  No selected key
    -> O_s = 0."""
    d = q.shape[-1]
    if len(keys) == 0:
        return np.zeros((len(rows), v.shape[-1]), dtype=F64)
    s = (q[rows] @ k[keys].T) / math.sqrt(d)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ v[keys]


def linear_branch(q, k, v, rows, keys, phi_kind="elu1"):
    """O_l = phi(Q) H / (phi(Q) Z) with H = sum phi(K_m)^T V_m and Z = sum phi(K_m)
    over the given (unselected) keys [SLA 关键设计 3], summed directly.  No key ->
    O_l = 0."""
    if len(keys) == 0:
        return np.zeros((len(rows), v.shape[-1]), dtype=F64)
    pk = phi(k[keys], phi_kind)
    Hm = pk.T @ v[keys]            # [d, dv]
    Z = pk.sum(axis=0)             # [d]
    pq = phi(q[rows], phi_kind)
    return (pq @ Hm) / (pq @ Z)[:, None]


def _blocks_to_do(B, H, nq, blocks):
    if blocks is None:
        return [(b, h, i) for b in range(B) for h in range(H) for i in range(nq)]
    return list(blocks)


def sla2_forward(q, k, v, kept, alpha, bq, bkv, phi_kind="elu1", blocks=None):
    """SLA2 output O = alpha*O_s + (1-alpha)*O_l [SLA2-deep §04, SLA2-sum §2.A],
    alpha per (batch, head, query block) as in the kernel description
    [SLA2-deep §08].  O_s runs over the kept key blocks, O_l over all others.

    q, k, v: float64 [B,H,N,d]; kept: int [B,H,nq,k]; alpha: [B,H,nq].
    blocks: optional list of (b,h,i) to compute (others stay NaN).
    Returns dict with "o", "o_s", "o_l" (float64 [B,H,N,d])."""
    B, H, N, d = q.shape
    nq = -(-N // bq)
    n_kv = -(-N // bkv)
    out = {n: np.full(v.shape, np.nan) for n in ("o", "o_s", "o_l")}
    for (b, h, i) in _blocks_to_do(B, H, nq, blocks):
        rows = _rows(i, bq, N)
        sel = sorted(int(j) for j in kept[b, h, i])
        uns = [j for j in range(n_kv) if j not in set(sel)]
        qs, ks, vs = q[b, h], k[b, h], v[b, h]
        o_s = sparse_branch(qs, ks, vs, rows, _tokens_of(sel, bkv, N))
        o_l = linear_branch(qs, ks, vs, rows, _tokens_of(uns, bkv, N), phi_kind)
        a = float(alpha[b, h, i])
        out["o_s"][b, h, rows] = o_s
        out["o_l"][b, h, rows] = o_l
        out["o"][b, h, rows] = a * o_s + (1.0 - a) * o_l
    return out


def sla_forward(q, k, v, labels, wproj, bq, bkv, phi_kind="elu1", blocks=None):
    """SLA output O = O_s + Proj(O_l) [SLA 关键设计 3]: sparse softmax over the
    critical blocks (+1), linear attention over the marginal blocks (0),
    negligible blocks (-1) skipped [SLA 关键设计 2].  Proj(x) = x @ wproj with
    wproj [d_in, d_out], no bias, shared by all heads.  Same layout as
    sla2_forward."""
    B, H, N, d = q.shape
    nq = -(-N // bq)
    wp = np.asarray(wproj, dtype=F64)
    out = {n: np.full(v.shape, np.nan) for n in ("o", "o_s", "o_l")}
    for (b, h, i) in _blocks_to_do(B, H, nq, blocks):
        rows = _rows(i, bq, N)
        lab = labels[b, h, i]
        crit = [int(j) for j in np.nonzero(lab == 1)[0]]
        marg = [int(j) for j in np.nonzero(lab == 0)[0]]
        qs, ks, vs = q[b, h], k[b, h], v[b, h]
        o_s = sparse_branch(qs, ks, vs, rows, _tokens_of(crit, bkv, N))
        o_l = linear_branch(qs, ks, vs, rows, _tokens_of(marg, bkv, N), phi_kind)
        out["o_s"][b, h, rows] = o_s
        out["o_l"][b, h, rows] = o_l
        out["o"][b, h, rows] = o_s + o_l @ wp
    return out


# ----------------------------------------------------------------------------
# FP8 e4m3 codec (OCP 8-bit floating point spec, E4M3: bias 7, no infinities,
# max finite 448, NaN = S.1111.111), round to nearest even, saturating.
# ----------------------------------------------------------------------------

def e4m3_encode(x32: np.ndarray) -> np.ndarray:
    """float32 -> uint8 e4m3 codes, round-to-nearest-even, finite values beyond
    448 saturate to +-448, NaN -> 0x7F with the sign bit."""
    x = np.asarray(x32, dtype=F32).astype(F64)
    sign = np.signbit(x).astype(np.uint8) << 7
    a = np.abs(x)
    code = np.zeros(x.shape, dtype=np.uint8)
    nan = np.isnan(a)
    sat = (~nan) & (a >= 448.0)
    sub = (~nan) & (~sat) & (a < 2.0 ** -6)
    nor = (~nan) & (~sat) & (~sub)
    # subnormals (and zero): multiples of 2^-9, code = m, m in 0..8 (8 -> min normal)
    m_sub = np.rint(a[sub] / 2.0 ** -9).astype(np.int64)
    code[sub] = m_sub.astype(np.uint8)
    # normals: a = f * 2^e with f in [1,2)
    fr, ex = np.frexp(a[nor])          # a = fr * 2^ex, fr in [0.5, 1)
    e = ex - 1
    f = fr * 2.0
    q = np.rint((f - 1.0) * 8.0).astype(np.int64)
    carry = q == 8
    e = np.where(carry, e + 1, e)
    q = np.where(carry, 0, q)
    big = e > 8                        # cannot happen for a < 448, kept for clarity
    c = ((e + 7) << 3) | q
    c = np.where(big, 0x7E, c)
    code[nor] = c.astype(np.uint8)
    code[sat] = 0x7E
    code[nan] = 0x7F
    return code | sign


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    """uint8 e4m3 codes -> float64 values."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return s * val


def e4m3_round(x32: np.ndarray) -> np.ndarray:
    """Value of x after an e4m3 round trip, float64."""
    return e4m3_decode(e4m3_encode(x32))


def int8_round(x32: np.ndarray) -> np.ndarray:
    """Value of x after a symmetric INT8 round trip, float64: round to the
    nearest integer (ties to even), saturate to [-127, 127]."""
    return np.clip(np.rint(np.asarray(x32, dtype=F64)), -127.0, 127.0)


# ----------------------------------------------------------------------------
# Low-bit (FP8 e4m3) sparse branch  [SLA2-deep §07]
#
# The page quantises Q and K, computes the low-bit Q K^T, dequantises and takes
# the softmax; quantises P and V, computes the low-bit P V and dequantises;
# before that K is smoothed by subtracting its column mean.  It does not fix
# the format or the scale granularity; the readings taken here:
#   - format e4m3 (OCP), round to nearest even, saturating;
#   - K smoothing: mu = mean of K over the valid tokens of (b,h), K' = K - mu
#     rounded to fp32 (a constant shift of every score in a row, which the
#     softmax ignores);
#   - Q and K': one scale per (b,h) and 128-token block: amax over the block,
#     inv = 448 / amax in fp32 (1 if amax = 0), x8 = e4m3(fp32(x * inv)),
#     scale = amax / 448 in fp32;
#   - V: one scale per (b,h) and channel over all valid tokens, same rule;
#   - P: online softmax over the kept blocks in ascending order, one kept
#     block at a time: after each block p = exp(S - m) with m the running row
#     max including that block, p8 = e4m3(fp32(p * 448)); the row sum uses
#     the unquantised p.  The page fixes no tile, so the block, the unit the
#     mask selects, is the tile here.  kv_tile > 1 groups that many
#     consecutive kept blocks per step instead; it exists only so a pin can
#     show that the grouping moves nothing but the rounding of P (without
#     quantisation online softmax is exact for any grouping).
# The page names "INT8 or FP8" and points to SageAttention2++ for the scheme
# without fixing it.  The INT8 variant read from that: Q and K' in INT8 with
# the same per-block rule (qmax 127 in place of 448, codes rint(x * inv) ties
# to even, saturated to +-127; their product is exact in integers), P and V
# in e4m3 as above.
# ----------------------------------------------------------------------------

def _e4m3_q(x32, codec):
    return codec(np.asarray(x32, dtype=F32))


def _quant_blocks(x32, blk, codec, qmax=448.0):
    """Per block of `blk` tokens (rows of x32 [n, d]): (decoded values, scales),
    codes of x * qmax / amax and scale amax / qmax (both fp32)."""
    n = x32.shape[0]
    vals = np.empty(x32.shape, dtype=F64)
    scales = []
    for t0 in range(0, n, blk):
        xb = x32[t0:t0 + blk]
        amax = F32(np.abs(xb).max()) if xb.size else F32(0.0)
        inv = F32(qmax) / amax if amax > 0 else F32(1.0)
        vals[t0:t0 + blk] = _e4m3_q(xb * inv, codec)
        scales.append(F64(F32(amax / F32(qmax))) if amax > 0 else F64(F32(1.0) / F32(qmax)))
    return vals, np.array(scales, dtype=F64)


def sla2_forward_fp8(q, k, v, kept, alpha, bq, bkv, phi_kind="elu1", blocks=None, codec=None, qblk=128,
                     kv_tile=1, qk_codec=None, qk_max=448.0):
    """SLA2 output with the low-bit sparse branch described above; the linear
    branch and the combine are the fp64 ones of sla2_forward.  q, k, v: exact
    values of the inputs as float64 [B,H,N,d].  codec(x32) -> float64 values
    after the e4m3 round trip (e4m3_round by default; an identity codec turns
    the quantisation off, which pins the bookkeeping to sla2_forward).
    qk_codec, qk_max: the round trip and code range of Q and K' (default: codec
    and 448; the INT8 variant passes int8_round and 127)."""
    codec = e4m3_round if codec is None else codec
    qk_codec = codec if qk_codec is None else qk_codec
    B, H, N, d = q.shape
    nq = -(-N // bq)
    n_kv = -(-N // bkv)
    out = {n: np.full(v.shape, np.nan) for n in ("o", "o_s", "o_l")}
    todo = _blocks_to_do(B, H, nq, blocks)
    heads = sorted({(b, h) for (b, h, _) in todo})
    for (b, h) in heads:
        qs, ks, vs = q[b, h], k[b, h], v[b, h]
        mu = ks.mean(axis=0)
        kp32 = (ks - mu).astype(F32)
        q8, sq = _quant_blocks(qs.astype(F32), qblk, qk_codec, qk_max)
        k8, sk = _quant_blocks(kp32, qblk, qk_codec, qk_max)
        v32 = vs.astype(F32)
        vamax = np.abs(v32).max(axis=0)
        vinv = np.where(vamax > 0, F32(448.0) / np.where(vamax > 0, vamax, F32(1.0)), F32(1.0)).astype(F32)
        v8 = _e4m3_q(v32 * vinv[None, :], codec)
        sv = np.where(vamax > 0, (vamax / F32(448.0)).astype(F32), F32(1.0) / F32(448.0)).astype(F64)
        vdq = v8 * sv[None, :]
        tok_q = np.arange(N) // qblk
        for (_, _, i) in [t for t in todo if (t[0], t[1]) == (b, h)]:
            rows = _rows(i, bq, N)
            sel = sorted(int(j) for j in kept[b, h, i])
            uns = [j for j in range(n_kv) if j not in set(sel)]
            m = np.full(len(rows), -np.inf)
            l = np.zeros(len(rows))
            acc = np.zeros((len(rows), v.shape[-1]))
            qdq = q8[rows] * sq[tok_q[rows]][:, None]
            for g0 in range(0, len(sel), kv_tile):
                keys = np.concatenate([_rows(j, bkv, N) for j in sel[g0:g0 + kv_tile]])
                kdq = k8[keys] * sk[tok_q[keys]][:, None]
                s = (qdq @ kdq.T) / math.sqrt(d)
                m_new = np.maximum(m, s.max(axis=1))
                corr = np.exp(m - m_new)
                p = np.exp(s - m_new[:, None])
                l = l * corr + p.sum(axis=1)
                p8 = _e4m3_q((p * 448.0).astype(F32), codec) / 448.0
                acc = acc * corr[:, None] + p8 @ vdq[keys]
                m = m_new
            o_s = acc / l[:, None] if sel else np.zeros((len(rows), v.shape[-1]))
            o_l = linear_branch(qs, ks, vs, rows, _tokens_of(uns, bkv, N), phi_kind)
            a = float(alpha[b, h, i])
            out["o_s"][b, h, rows] = o_s
            out["o_l"][b, h, rows] = o_l
            out["o"][b, h, rows] = a * o_s + (1.0 - a) * o_l
    return out


def sla2_forward_int8(q, k, v, kept, alpha, bq, bkv, phi_kind="elu1", blocks=None, qblk=128, kv_tile=1):
    """SLA2 output with the INT8 variant of the low-bit branch: Q and K' in
    INT8 (int8_round, qmax 127, one scale per qblk-token block), P and V in
    e4m3 as in sla2_forward_fp8."""
    return sla2_forward_fp8(q, k, v, kept, alpha, bq, bkv, phi_kind, blocks, None, qblk, kv_tile,
                            qk_codec=int8_round, qk_max=127.0)


# ----------------------------------------------------------------------------
# Backward (fp64): gradients of sla2_forward / sla_forward with the block mask
# held fixed.  [SLA 关键设计 4]: the sparse part returns dQ, dK, dV the way
# FlashAttention does; the linear part follows the chain rule through dH_i and
# dZ_i, formed per query block and then spread over the keys that built H_i
# and Z_i.  [SLA2-deep §07], [SLA2-sum §2.C]: gradients are taken on the
# original, unquantised inputs, so the low-bit forward has no backward of its
# own.  The hard Top-k passes no gradient to the router; the stage that trains
# the router uses SoftTop-k instead [SLA2-deep §06].
# ----------------------------------------------------------------------------

def phi_backward(x, dphi, kind="elu1"):
    """dL/dx from dL/dphi(x) for the feature map phi above.  "elu1": phi'(x) is
    1 for x > 0 and exp(x) otherwise.  "softmax" over the channels of a token:
    dx = phi * (dphi - sum_c dphi_c phi_c)."""
    x = np.asarray(x, dtype=F64)
    if kind == "elu1":
        return dphi * np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))
    if kind == "softmax":
        p = phi(x, "softmax")
        return p * (dphi - (dphi * p).sum(axis=-1, keepdims=True))
    raise ValueError(kind)


def sparse_branch_backward(q, k, v, rows, keys, do_s):
    """Gradients of sparse_branch's O_s for the given rows over the selected
    keys.  With P the row softmax of S = Q K^T / sqrt(d) and O_s = P V:
      dV = P^T dO_s,  dP = dO_s V^T,  D = rowsum(dO_s * O_s),
      dS = P * (dP - D),  dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d).
    No selected key -> O_s = 0 and nothing flows.
    Returns (dq [rows, d], dk [keys, d], dv [keys, dv])."""
    d = q.shape[-1]
    if len(keys) == 0:
        return np.zeros((len(rows), d)), np.zeros((0, d)), np.zeros((0, v.shape[-1]))
    s = (q[rows] @ k[keys].T) / math.sqrt(d)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p = p / p.sum(axis=1, keepdims=True)
    o = p @ v[keys]
    dv = p.T @ do_s
    dp = do_s @ v[keys].T
    D = (do_s * o).sum(axis=1, keepdims=True)
    ds = p * (dp - D)
    dq = ds @ k[keys] / math.sqrt(d)
    dk = ds.T @ q[rows] / math.sqrt(d)
    return dq, dk, dv


def linear_branch_backward(q, k, v, rows, keys, do_l, phi_kind="elu1"):
    """Gradients of linear_branch's O_l = phi(Q) H / (phi(Q) Z) for the given
    rows over the given (unselected) keys, through dH and dZ:
      a = phi(q), num = a H, den = a . Z, O_l = num / den;
      dnum = dO_l / den,  dden = -rowsum(dO_l * O_l) / den;
      dphi(q) = dnum H^T + dden Z^T;
      dH = a^T dnum,  dZ = a^T dden  (sums over the rows);
      dphi(k_m) = dH v_m + dZ,  dv_m = dH^T phi(k_m)  for every key m;
    then dq and dk through phi_backward.  No key -> O_l = 0 and nothing flows.
    Returns (dq [rows, d], dk [keys, d], dv [keys, dv])."""
    if len(keys) == 0:
        return np.zeros((len(rows), q.shape[-1])), np.zeros((0, k.shape[-1])), np.zeros((0, v.shape[-1]))
    pk = phi(k[keys], phi_kind)
    Hm = pk.T @ v[keys]            # [d, dv]
    Z = pk.sum(axis=0)             # [d]
    pq = phi(q[rows], phi_kind)
    num = pq @ Hm
    den = pq @ Z
    o = num / den[:, None]
    dnum = do_l / den[:, None]
    dden = -(do_l * o).sum(axis=1) / den
    dpq = dnum @ Hm.T + dden[:, None] * Z[None, :]
    dH = pq.T @ dnum               # [d, dv]
    dZ = pq.T @ dden               # [d]
    dpk = v[keys] @ dH.T + dZ[None, :]
    dv = pk @ dH
    return phi_backward(q[rows], dpq, phi_kind), phi_backward(k[keys], dpk, phi_kind), dv


def sla2_backward(q, k, v, kept, alpha, do, bq, bkv, phi_kind="elu1", blocks=None):
    """Gradients of sla2_forward's O = alpha*O_s + (1-alpha)*O_l for the
    upstream gradient do [B,H,N,d], the mask held fixed:
      dO_s = alpha dO,  dO_l = (1 - alpha) dO,
      dalpha_i = sum over the rows of query block i of dO * (O_s - O_l).
    A key's gradient adds up over every query block that reads it: through the
    sparse branch where its block is kept, through the linear branch elsewhere.
    blocks: optional list of (b,h,i) whose share to add (default: all, which
    gives the full gradients).
    Returns dict dq, dk, dv (float64 [B,H,N,d]) and dalpha ([B,H,nq])."""
    B, H, N, d = q.shape
    nq = -(-N // bq)
    n_kv = -(-N // bkv)
    dq, dk, dv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    dalpha = np.zeros((B, H, nq))
    for (b, h, i) in _blocks_to_do(B, H, nq, blocks):
        qs, ks, vs = q[b, h], k[b, h], v[b, h]
        rows = _rows(i, bq, N)
        sel = sorted(int(j) for j in kept[b, h, i])
        uns = [j for j in range(n_kv) if j not in set(sel)]
        ts, tl = _tokens_of(sel, bkv, N), _tokens_of(uns, bkv, N)
        a = float(alpha[b, h, i])
        g = do[b, h, rows]
        o_s = sparse_branch(qs, ks, vs, rows, ts)
        o_l = linear_branch(qs, ks, vs, rows, tl, phi_kind)
        dalpha[b, h, i] = (g * (o_s - o_l)).sum()
        gq, gk, gv = sparse_branch_backward(qs, ks, vs, rows, ts, a * g)
        dq[b, h, rows] += gq
        dk[b, h, ts] += gk
        dv[b, h, ts] += gv
        gq, gk, gv = linear_branch_backward(qs, ks, vs, rows, tl, (1.0 - a) * g, phi_kind)
        dq[b, h, rows] += gq
        dk[b, h, tl] += gk
        dv[b, h, tl] += gv
    return {"dq": dq, "dk": dk, "dv": dv, "dalpha": dalpha}


def sla_backward(q, k, v, labels, wproj, do, bq, bkv, phi_kind="elu1", blocks=None):
    """Gradients of sla_forward's O = O_s + O_l Wp for the upstream gradient do,
    the labels held fixed:  dO_s = dO,  dO_l = dO Wp^T,  dWp = sum over every
    row of every head of O_l^T dO (Wp is shared).  Critical blocks (+1) take
    the sparse branch, marginal ones (0) the linear branch, negligible ones
    (-1) get no gradient.  blocks: optional list of (b,h,i) whose share to add
    (default: all, which gives the full gradients).
    Returns dict dq, dk, dv and dwproj ([d_in, d_out])."""
    B, H, N, d = q.shape
    nq = -(-N // bq)
    wp = np.asarray(wproj, dtype=F64)
    dq, dk, dv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    dwp = np.zeros(wp.shape)
    for (b, h, i) in _blocks_to_do(B, H, nq, blocks):
        qs, ks, vs = q[b, h], k[b, h], v[b, h]
        rows = _rows(i, bq, N)
        lab = labels[b, h, i]
        tc = _tokens_of([int(j) for j in np.nonzero(lab == 1)[0]], bkv, N)
        tm = _tokens_of([int(j) for j in np.nonzero(lab == 0)[0]], bkv, N)
        g = do[b, h, rows]
        o_l = linear_branch(qs, ks, vs, rows, tm, phi_kind)
        dwp += o_l.T @ g
        gq, gk, gv = sparse_branch_backward(qs, ks, vs, rows, tc, g)
        dq[b, h, rows] += gq
        dk[b, h, tc] += gk
        dv[b, h, tc] += gv
        gq, gk, gv = linear_branch_backward(qs, ks, vs, rows, tm, g @ wp.T, phi_kind)
        dq[b, h, rows] += gq
        dk[b, h, tm] += gk
        dv[b, h, tm] += gv
    return {"dq": dq, "dk": dk, "dv": dv, "dwproj": dwp}
