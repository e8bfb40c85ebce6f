"""The decomposition the GPU backward is built on (sparse_linear_attention_b200/
csrc/backward.cu, header comment) restated in numpy and checked against the
oracle's sla2_backward, on the CPU.

The kernel writes the linear branch as totals minus the kept blocks: H_i =
H_tot - sum_kept phi(K_j)^T V_j, and the gradient that H_i, Z_i send to the
unselected keys as (dH_tot, dZ_tot) minus the kept blocks' share.  It also
recomputes the softmax in three passes over the kept blocks (row max; row sum,
O_s, num, den; gradients) per 32-row tile.  This restatement follows those
steps and shares no code with the kernel or the oracle; agreement to rounding
shows the algebra is exact, including k = 0, k = n_kv, ragged blocks and both
feature maps ("SLA: Beyond Sparsity …" (papernotes.org) 关键设计 4).

The same decomposition for SLA's three labels (critical blocks in the softmax,
critical and negligible blocks both taken out of the linear totals, the
W_proj gradient) is checked against the oracle's sla_backward; backward.cu
follows it for SLA.

Rearrangements of the SLA2 decomposition follow: a key-major one, the
arrangement of the tensor-core kernels (csrc/backward_tc.cu: statistics from
the attention kernel, query-major dQ, per-tile dH_i partials, power-of-two
scalings), and the key side regrouped through those partials; then the same
regrouping for SLA's three labels, which a tensor-core SLA backward would
follow.  Each is checked in fp64 against the oracle.
"""
import math

import numpy as np
import pytest

from oracle import sla_oracle as orc


def _phi(x, kind):
    if kind == "elu1":
        return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))
    e = np.exp(x - x.max(-1, keepdims=True))
    return e / e.sum(-1, keepdims=True)


def _phi_grad(x, g, kind):
    if kind == "elu1":
        return g * np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))
    f = _phi(x, kind)
    return f * (g - (g * f).sum(-1, keepdims=True))


def _decomposed(q, k, v, kept, alpha, do, bq, bkv, kind):
    B, H, N, d = q.shape
    nq, nkv = -(-N // bq), -(-N // bkv)
    sc = 1.0 / math.sqrt(d)
    dq, dk, dv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    dal = np.zeros((B, H, nq))
    has_lin = kept.shape[-1] < nkv
    for b in range(B):
        for h in range(H):
            Q, K, V, G = q[b, h], k[b, h], v[b, h], do[b, h]
            PK = _phi(K, kind)
            Ht, Zt = PK.T @ V, PK.sum(0)
            dHt, dZt, dPK = np.zeros((d, d)), np.zeros(d), np.zeros((N, d))
            for i in range(nq):
                a = alpha[b, h, i]
                blocks = [np.arange(j * bkv, min((j + 1) * bkv, N)) for j in kept[b, h, i]]
                for r0 in range(i * bq, min((i + 1) * bq, N), 32):
                    rows = np.arange(r0, min(r0 + 32, N))
                    Qt, Gt = Q[rows], G[rows]
                    PQ = _phi(Qt, kind)
                    num = PQ @ Ht
                    m = np.full(len(rows), -np.inf)
                    for ks in blocks:
                        m = np.maximum(m, (sc * Qt @ K[ks].T).max(1))
                    l, oacc, rsa = np.zeros(len(rows)), np.zeros((len(rows), d)), np.zeros(len(rows))
                    for ks in blocks:
                        P = np.exp(sc * Qt @ K[ks].T - m[:, None])
                        A = PQ @ PK[ks].T
                        l += P.sum(1)
                        oacc += P @ V[ks]
                        num -= A @ V[ks]
                        rsa += A.sum(1)
                    Os = oacc / l[:, None] if blocks else np.zeros_like(oacc)
                    if has_lin:
                        den = PQ @ Zt - rsa
                        Ol = num / den[:, None]
                        s = (1.0 - a) / den
                        dd = -(1.0 - a) * (Gt * Ol).sum(1) / den
                    else:
                        Ol, s, dd = np.zeros_like(Os), np.zeros(len(rows)), np.zeros(len(rows))
                    D = a * (Gt * Os).sum(1)
                    dal[b, h, i] += (Gt * (Os - Ol)).sum()
                    dqs, dpq = np.zeros((len(rows), d)), np.zeros((len(rows), d))
                    for ks in blocks:
                        P = np.exp(sc * Qt @ K[ks].T - m[:, None]) / l[:, None]
                        A = PQ @ PK[ks].T
                        Gk = Gt @ V[ks].T
                        dS = P * (a * Gk - D[:, None])
                        C = a * P - s[:, None] * A
                        Bx = s[:, None] * Gk + dd[:, None]
                        dqs += dS @ K[ks]
                        dpq -= Bx @ PK[ks]
                        dk[b, h, ks] += sc * dS.T @ Qt
                        dv[b, h, ks] += C.T @ Gt
                        if has_lin:
                            dPK[ks] -= Bx.T @ PQ
                    if has_lin:
                        dpq += s[:, None] * (Gt @ Ht.T) + dd[:, None] * Zt[None, :]
                        dHt += PQ.T @ (s[:, None] * Gt)
                        dZt += PQ.T @ dd
                    dq[b, h, rows] = sc * dqs + _phi_grad(Qt, dpq, kind)
            dPK += V @ dHt.T + dZt[None, :]
            dv[b, h] += PK @ dHt
            dk[b, h] += _phi_grad(K, dPK, kind)
    return {"dq": dq, "dk": dk, "dv": dv, "dalpha": dal}


@pytest.mark.parametrize("N,d,bq,kk,kind", [(200, 16, 64, 2, "elu1"), (333, 8, 128, 3, "softmax"),
                                            (130, 16, 64, 0, "elu1"), (130, 16, 64, 3, "elu1"),
                                            (97, 8, 64, 2, "softmax")])
def test_decomposition_matches_oracle(N, d, bq, kk, kind):
    rng = np.random.default_rng(N + kk)
    H, bkv = 2, 64
    q, k, v, do = (rng.standard_normal((1, H, N, d)) for _ in range(4))
    nq, nkv = -(-N // bq), -(-N // bkv)
    kk = min(kk, nkv)
    kept = np.array([[[np.sort(rng.choice(nkv, kk, replace=False)) for _ in range(nq)] for _ in range(H)]])
    kept = kept.reshape(1, H, nq, kk)
    alpha = rng.uniform(0.1, 0.9, (1, H, nq))
    ref = orc.sla2_backward(q, k, v, kept, alpha, do, bq, bkv, kind)
    got = _decomposed(q, k, v, kept, alpha, do, bq, bkv, kind)
    for name in ref:
        assert np.allclose(got[name], ref[name], atol=1e-12, rtol=1e-10), name


def _decomposed_sla(q, k, v, labels, wp, do, bq, bkv, kind):
    """SLA (O = O_s + O_l W_proj): the sparse passes run over the critical
    blocks; the linear branch is the totals minus the critical AND the
    negligible blocks (both leave it), so the kept share that goes back to the
    keys is taken over both lists; dO_s = dO, dO_l = dO W_proj^T, and
    dW_proj = sum O_l^T dO."""
    B, H, N, d = q.shape
    nq, nkv = -(-N // bq), -(-N // bkv)
    sc = 1.0 / math.sqrt(d)
    dq, dk, dv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    dwp = np.zeros(wp.shape)
    for b in range(B):
        for h in range(H):
            Q, K, V, G = q[b, h], k[b, h], v[b, h], do[b, h]
            PK = _phi(K, kind)
            Ht, Zt = PK.T @ V, PK.sum(0)
            dHt, dZt, dPK = np.zeros((d, d)), np.zeros(d), np.zeros((N, d))
            for i in range(nq):
                lab = labels[b, h, i]
                crit = [np.arange(j * bkv, min((j + 1) * bkv, N)) for j in np.nonzero(lab == 1)[0]]
                out = [np.arange(j * bkv, min((j + 1) * bkv, N)) for j in np.nonzero(lab != 0)[0]]
                has_lin = (lab == 0).any()
                for r0 in range(i * bq, min((i + 1) * bq, N), 32):
                    rows = np.arange(r0, min(r0 + 32, N))
                    Qt, Gs = Q[rows], G[rows]
                    Gl = Gs @ wp.T
                    PQ = _phi(Qt, kind)
                    num, rsa = PQ @ Ht, np.zeros(len(rows))
                    for ks in out:
                        A = PQ @ PK[ks].T
                        num -= A @ V[ks]
                        rsa += A.sum(1)
                    m = np.full(len(rows), -np.inf)
                    for ks in crit:
                        m = np.maximum(m, (sc * Qt @ K[ks].T).max(1))
                    l, oacc = np.zeros(len(rows)), np.zeros((len(rows), d))
                    for ks in crit:
                        P = np.exp(sc * Qt @ K[ks].T - m[:, None])
                        l += P.sum(1)
                        oacc += P @ V[ks]
                    Os = oacc / l[:, None] if crit else np.zeros_like(oacc)
                    if has_lin:
                        den = PQ @ Zt - rsa
                        Ol = num / den[:, None]
                        s = 1.0 / den
                        dd = -(Gl * Ol).sum(1) / den
                    else:
                        Ol, s, dd = np.zeros_like(Os), np.zeros(len(rows)), np.zeros(len(rows))
                    dwp += Ol.T @ Gs
                    D = (Gs * Os).sum(1)
                    dqs, dpq = np.zeros((len(rows), d)), np.zeros((len(rows), d))
                    for ks in crit:
                        P = np.exp(sc * Qt @ K[ks].T - m[:, None]) / l[:, None]
                        dS = P * (Gs @ V[ks].T - D[:, None])
                        dqs += dS @ K[ks]
                        dk[b, h, ks] += sc * dS.T @ Qt
                        dv[b, h, ks] += P.T @ Gs
                    if has_lin:
                        for ks in out:
                            A = PQ @ PK[ks].T
                            Bx = s[:, None] * (Gl @ V[ks].T) + dd[:, None]
                            dpq -= Bx @ PK[ks]
                            dv[b, h, ks] -= (s[:, None] * A).T @ Gl
                            dPK[ks] -= Bx.T @ PQ
                        dpq += s[:, None] * (Gl @ Ht.T) + dd[:, None] * Zt[None, :]
                        dHt += PQ.T @ (s[:, None] * Gl)
                        dZt += PQ.T @ dd
                    dq[b, h, rows] = sc * dqs + _phi_grad(Qt, dpq, kind)
            dPK += V @ dHt.T + dZt[None, :]
            dv[b, h] += PK @ dHt
            dk[b, h] += _phi_grad(K, dPK, kind)
    return {"dq": dq, "dk": dk, "dv": dv, "dwproj": dwp}


@pytest.mark.parametrize("N,d,bq,kind,n_crit,n_negl", [(200, 16, 64, "elu1", 1, 1), (333, 8, 128, "softmax", 2, 1),
                                                        (130, 16, 64, "elu1", 0, 1), (130, 16, 64, "elu1", 2, 1),
                                                        (130, 16, 64, "elu1", 3, 0)])
def test_sla_decomposition_matches_oracle(N, d, bq, kind, n_crit, n_negl):
    """Critical, marginal and negligible blocks; no critical block; no marginal
    block (critical and negligible fill the row); every block critical."""
    rng = np.random.default_rng(N + 10 * n_crit + n_negl)
    H, bkv = 2, 64
    q, k, v, do = (rng.standard_normal((1, H, N, d)) for _ in range(4))
    nq, nkv = -(-N // bq), -(-N // bkv)
    labels = np.zeros((1, H, nq, nkv), dtype=np.int8)
    for h, i in np.ndindex(H, nq):
        perm = rng.permutation(nkv)
        labels[0, h, i, perm[:n_crit]] = 1
        labels[0, h, i, perm[n_crit:n_crit + n_negl]] = -1
    wp = rng.standard_normal((d, d)) / math.sqrt(d)
    ref = orc.sla_backward(q, k, v, labels, wp, do, bq, bkv, kind)
    got = _decomposed_sla(q, k, v, labels, wp, do, bq, bkv, kind)
    for name in ref:
        assert np.allclose(got[name], ref[name], atol=1e-12, rtol=1e-10), name


def _key_major(q, k, v, kept, alpha, do, bq, bkv, kind):
    """The SLA2 backward restructured key-major: a query-major pass keeps per
    row only the log-sum-exp of the kept scores, D, s and dden (and forms dH_tot,
    dZ_tot and the linear dQ terms); then, per key block, the query blocks that
    keep it (the inverse map of the kept lists, ascending) give
      G^T = V dO^T,  dS^T = P^T * (alpha G^T - D),  C^T = alpha P^T - s A^T,
      dK += dS^T Q / sqrt(d),  dV += C^T dO,  dphi(K) -= Bx^T phi(Q),
    and dQ += dS K / sqrt(d) - Bx phi(K) is scattered back (Bx = s G + dden)."""
    B, H, N, d = q.shape
    nq, nkv = -(-N // bq), -(-N // bkv)
    sc = 1.0 / math.sqrt(d)
    dq, dk, dv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    dal = np.zeros((B, H, nq))
    has_lin = kept.shape[-1] < nkv
    for b in range(B):
        for h in range(H):
            Q, K, V, G = q[b, h], k[b, h], v[b, h], do[b, h]
            PK, PQ = _phi(K, kind), _phi(Q, kind)
            Ht, Zt = PK.T @ V, PK.sum(0)
            keys_of = [np.arange(j * bkv, min((j + 1) * bkv, N)) for j in range(nkv)]
            lse, D, s, dd = np.zeros(N), np.zeros(N), np.zeros(N), np.zeros(N)
            dHt, dZt, dPK = np.zeros((d, d)), np.zeros(d), np.zeros((N, d))
            dpq_all = np.zeros((N, d))  # dphi(Q) from the totals; the kept share is added key-major
            for i in range(nq):  # query-major statistics
                rows = np.arange(i * bq, min((i + 1) * bq, N))
                a = alpha[b, h, i]
                ks = np.concatenate([keys_of[j] for j in kept[b, h, i]]) if kept.shape[-1] else np.zeros(0, int)
                if len(ks):
                    S = sc * Q[rows] @ K[ks].T
                    mx = S.max(1)
                    lse[rows] = mx + np.log(np.exp(S - mx[:, None]).sum(1))
                    Os = np.exp(S - lse[rows][:, None]) @ V[ks]
                else:
                    Os = np.zeros((len(rows), d))
                if has_lin:
                    A = PQ[rows] @ PK[ks].T if len(ks) else np.zeros((len(rows), 0))
                    den = PQ[rows] @ Zt - A.sum(1)
                    Ol = (PQ[rows] @ Ht - A @ V[ks]) / den[:, None]
                    s[rows] = (1 - a) / den
                    dd[rows] = -(1 - a) * (G[rows] * Ol).sum(1) / den
                else:
                    Ol = np.zeros_like(Os)
                D[rows] = a * (G[rows] * Os).sum(1)
                dal[b, h, i] = (G[rows] * (Os - Ol)).sum()
                dpq_all[rows] = s[rows][:, None] * (G[rows] @ Ht.T) + dd[rows][:, None] * Zt[None, :]
                if has_lin:
                    dHt += PQ[rows].T @ (s[rows][:, None] * G[rows])
                    dZt += PQ[rows].T @ dd[rows]
            users = [[i for i in range(nq) if j in set(int(x) for x in kept[b, h, i])] for j in range(nkv)]
            dpq_kept = np.zeros((N, d))
            dqs = np.zeros((N, d))
            for j in range(nkv):  # key-major
                ks = keys_of[j]
                for i in users[j]:
                    rows = np.arange(i * bq, min((i + 1) * bq, N))
                    a = alpha[b, h, i]
                    PT = np.exp(sc * K[ks] @ Q[rows].T - lse[rows][None, :])
                    AT = PK[ks] @ PQ[rows].T
                    GT = V[ks] @ G[rows].T
                    dST = PT * (a * GT - D[rows][None, :])
                    CT = a * PT - AT * s[rows][None, :]
                    BxT = GT * s[rows][None, :] + dd[rows][None, :]
                    dk[b, h, ks] += sc * dST @ Q[rows]
                    dv[b, h, ks] += CT @ G[rows]
                    if has_lin:
                        dPK[ks] -= BxT @ PQ[rows]
                        dpq_kept[rows] -= BxT.T @ PK[ks]
                    dqs[rows] += sc * dST.T @ K[ks]
            dq[b, h] = dqs + _phi_grad(Q, dpq_all + dpq_kept, kind)
            dPK += V @ dHt.T + dZt[None, :]
            dv[b, h] += PK @ dHt
            dk[b, h] += _phi_grad(K, dPK, kind)
    return {"dq": dq, "dk": dk, "dv": dv, "dalpha": dal}


@pytest.mark.parametrize("N,d,bq,kk,kind", [(200, 16, 64, 2, "elu1"), (333, 8, 128, 3, "softmax"),
                                            (130, 16, 64, 0, "elu1"), (130, 16, 64, 3, "elu1")])
def test_key_major_restatement_matches_oracle(N, d, bq, kk, kind):
    rng = np.random.default_rng(7 * N + kk)
    H, bkv = 2, 64
    q, k, v, do = (rng.standard_normal((1, H, N, d)) for _ in range(4))
    nq, nkv = -(-N // bq), -(-N // bkv)
    kk = min(kk, nkv)
    kept = np.array([[[np.sort(rng.choice(nkv, kk, replace=False)) for _ in range(nq)] for _ in range(H)]])
    kept = kept.reshape(1, H, nq, kk)
    alpha = rng.uniform(0.1, 0.9, (1, H, nq))
    ref = orc.sla2_backward(q, k, v, kept, alpha, do, bq, bkv, kind)
    got = _key_major(q, k, v, kept, alpha, do, bq, bkv, kind)
    for name in ref:
        assert np.allclose(got[name], ref[name], atol=1e-12, rtol=1e-10), name


def _tensor_core_arrangement(q, k, v, kept, alpha, do, bq, bkv, kind):
    """The arrangement of sparse_linear_attention_b200/csrc/backward_tc.cu, in
    fp64: per-row statistics as the attention kernel's epilogue writes them
    (log2-sum-exp from a stale running max, D, s, dden, the row's dalpha share);
    a query-major dQ pass with Bx and s dO scaled by the power of two sigma >=
    max Z_tot and H_tot entering as H_tot / sigma, which also forms the per-tile
    dH_i, dZ_i; a key-major pass over the inverse lists accumulating the
    transposed key-side products; dH_tot, dZ_tot as sums of the tile partials;
    the per-key step with dH_tot scaled by the power of two tau."""
    B, H, N, d = q.shape
    nq, nkv = -(-N // bq), -(-N // bkv)
    sc = 1.0 / math.sqrt(d)
    l2e = 1.0 / math.log(2.0)
    kk = kept.shape[-1]
    dq, dk, dv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    dal = np.zeros((B, H, nq))
    for b in range(B):
        for h in range(H):
            Q, K, V, G = q[b, h], k[b, h], v[b, h], do[b, h]
            PK, PQ = _phi(K, kind), _phi(Q, kind)
            Ht, Zt = PK.T @ V, PK.sum(0)
            sigma = 2.0 ** math.ceil(math.log2(max(Zt.max(), 1e-300)))
            keys_of = [np.arange(j * bkv, min((j + 1) * bkv, N)) for j in range(nkv)]
            stats = np.zeros((N, 5))
            # 1. the attention kernel's statistics epilogue
            for i in range(nq):
                rows = np.arange(i * bq, min((i + 1) * bq, N))
                a = alpha[b, h, i]
                ks = np.concatenate([keys_of[j] for j in kept[b, h, i]]) if kk else np.zeros(0, int)
                Os, Ol = np.zeros((len(rows), d)), np.zeros((len(rows), d))
                lse2 = np.zeros(len(rows))
                if len(ks):
                    S2 = sc * l2e * (Q[rows] @ K[ks].T)
                    m = S2.max(1) - 3.0  # a stale running max: lse2 does not depend on it
                    p = np.exp2(S2 - m[:, None])
                    lse2 = m + np.log2(p.sum(1))
                    Os = (p @ V[ks]) / p.sum(1)[:, None]
                lin = kk < nkv
                s_r, dd_r = np.zeros(len(rows)), np.zeros(len(rows))
                if lin:
                    A = PQ[rows] @ PK[ks].T if len(ks) else np.zeros((len(rows), 0))
                    den = PQ[rows] @ Zt - A.sum(1)
                    Ol = (PQ[rows] @ Ht - A @ V[ks]) / den[:, None]
                    s_r = (1 - a) / den
                    dd_r = -(1 - a) * (G[rows] * Ol).sum(1) / den
                stats[rows] = np.stack([lse2, a * (G[rows] * Os).sum(1), s_r, dd_r,
                                        (G[rows] * (Os - Ol)).sum(1)], axis=1)
                dal[b, h, i] = stats[rows, 4].sum()
            users = [[i for i in range(nq) if j in set(int(x) for x in kept[b, h, i])] for j in range(nkv)]
            dh_parts, dz_parts = [], []
            # 2. query-major dQ, per-tile dH_i, dZ_i
            for i in range(nq):
                rows = np.arange(i * bq, min((i + 1) * bq, N))
                a = alpha[b, h, i]
                lse2, D, s_r, dd_r = (stats[rows, c] for c in range(4))
                dqs, dql = np.zeros((len(rows), d)), np.zeros((len(rows), d))
                for j in kept[b, h, i]:
                    ks = keys_of[j]
                    P = np.exp2(sc * l2e * (Q[rows] @ K[ks].T) - lse2[:, None])
                    Gm = G[rows] @ V[ks].T
                    dS = P * (a * Gm - D[:, None])
                    nbx = -(s_r[:, None] * Gm + dd_r[:, None]) * sigma
                    dqs += dS @ K[ks]
                    dql += nbx @ PK[ks]
                ssd = (s_r * sigma)[:, None] * G[rows]
                hterm = ssd @ (Ht / sigma).T
                dh_parts.append(PQ[rows].T @ ssd / sigma)
                dz_parts.append(PQ[rows].T @ dd_r)
                gphi = dql / sigma + hterm + dd_r[:, None] * Zt[None, :]
                dq[b, h, rows] = sc * dqs + _phi_grad(Q[rows], gphi, kind)
            # 3. key-major kept shares (transposed accumulators)
            dphik = np.zeros((N, d))
            for j in range(nkv):
                ks = keys_of[j]
                dVT, dKT, dPT = np.zeros((d, len(ks))), np.zeros((d, len(ks))), np.zeros((d, len(ks)))
                for i in users[j]:
                    rows = np.arange(i * bq, min((i + 1) * bq, N))
                    a = alpha[b, h, i]
                    lse2, D, s_r, dd_r = (stats[rows, c] for c in range(4))
                    P = np.exp2(sc * l2e * (Q[rows] @ K[ks].T) - lse2[:, None])
                    Gm = G[rows] @ V[ks].T
                    A = PQ[rows] @ PK[ks].T
                    dS = P * (a * Gm - D[:, None])
                    C = a * P - s_r[:, None] * A
                    nbx = -(s_r[:, None] * Gm + dd_r[:, None]) * sigma
                    dVT += G[rows].T @ C
                    dKT += Q[rows].T @ dS
                    dPT += PQ[rows].T @ nbx
                dv[b, h, ks] = dVT.T
                dk[b, h, ks] = sc * dKT.T
                dphik[ks] = dPT.T / sigma
            # 4. totals: the tile partials summed, tau, the per-key step
            dHt = np.sum(dh_parts, axis=0)
            dZt = np.sum(dz_parts, axis=0)
            mh = np.abs(dHt).max()
            tau = 2.0 ** (14 - math.frexp(mh)[1]) if mh > 0 else 1.0
            acc1 = V @ (tau * dHt).T
            acc2 = PK @ (tau * dHt)
            dphi = acc1 / tau + dZt[None, :] + dphik
            dk[b, h] += _phi_grad(K, dphi, kind)
            dv[b, h] += acc2 / tau
    return {"dq": dq, "dk": dk, "dv": dv, "dalpha": dal}


@pytest.mark.parametrize("N,d,bq,kk,kind", [(300, 16, 128, 2, "elu1"), (333, 8, 128, 3, "softmax"),
                                            (130, 16, 128, 0, "elu1"), (256, 16, 128, 4, "elu1"),
                                            (100, 8, 128, 1, "softmax")])
def test_tensor_core_arrangement_matches_oracle(N, d, bq, kk, kind):
    """The tensor-core backward's order of work and its exact power-of-two
    scalings reproduce the oracle's gradients in fp64 (k = 0, k = n_kv, ragged
    tiles, both feature maps)."""
    rng = np.random.default_rng(11 * N + kk)
    H, bkv = 2, 64
    q, k, v, do = (rng.standard_normal((1, H, N, d)) for _ in range(4))
    nq, nkv = -(-N // bq), -(-N // bkv)
    kk = min(kk, nkv)
    kept = np.array([[[np.sort(rng.choice(nkv, kk, replace=False)) for _ in range(nq)] for _ in range(H)]])
    kept = kept.reshape(1, H, nq, kk)
    alpha = rng.uniform(0.1, 0.9, (1, H, nq))
    ref = orc.sla2_backward(q, k, v, kept, alpha, do, bq, bkv, kind)
    got = _tensor_core_arrangement(q, k, v, kept, alpha, do, bq, bkv, kind)
    for name in ref:
        assert np.allclose(got[name], ref[name], atol=1e-12, rtol=1e-10), name


def _key_block_linear_from_tile_partials(q, k, v, kept, alpha, do, bq, bkv, kind):
    """The key side regrouped around the query tiles' linear partials: with
    dH_i = phi(Q_i)^T (s dO_i) and dZ_i = phi(Q_i)^T dden_i per query tile i and
    M_j = dH_tot - sum over the tiles i keeping key block j of dH_i,
      dV_j    = sum_i (alpha_i P_ij)^T dO_i + phi(K_j) M_j
      dphi(K_j) = V_j M_j^T + dZ_tot - sum_i dZ_i
      dK_j    = sum_i dS_ij^T Q_i / sqrt(d) + phi'(K_j) dphi(K_j)
    so the key-major pass needs only S, G, dS and P; the linear part comes from
    the partials.  dQ as before (query-major)."""
    B, H, N, d = q.shape
    nq, nkv = -(-N // bq), -(-N // bkv)
    sc = 1.0 / math.sqrt(d)
    kk = kept.shape[-1]
    base = _tensor_core_arrangement(q, k, v, kept, alpha, do, bq, bkv, kind)  # dq, dalpha
    dk, dv = np.zeros(k.shape), np.zeros(v.shape)
    for b in range(B):
        for h in range(H):
            Q, K, V, G = q[b, h], k[b, h], v[b, h], do[b, h]
            PK, PQ = _phi(K, kind), _phi(Q, kind)
            Ht, Zt = PK.T @ V, PK.sum(0)
            keys_of = [np.arange(j * bkv, min((j + 1) * bkv, N)) for j in range(nkv)]
            lse, D, s, dd = np.zeros(N), np.zeros(N), np.zeros(N), np.zeros(N)
            dH_i, dZ_i = [], []
            for i in range(nq):
                rows = np.arange(i * bq, min((i + 1) * bq, N))
                a = alpha[b, h, i]
                ks = np.concatenate([keys_of[j] for j in kept[b, h, i]]) if kk else np.zeros(0, int)
                Os = np.zeros((len(rows), d))
                if len(ks):
                    S = sc * Q[rows] @ K[ks].T
                    mx = S.max(1)
                    lse[rows] = mx + np.log(np.exp(S - mx[:, None]).sum(1))
                    Os = np.exp(S - lse[rows][:, None]) @ V[ks]
                if kk < nkv:
                    A = PQ[rows] @ PK[ks].T if len(ks) else np.zeros((len(rows), 0))
                    den = PQ[rows] @ Zt - A.sum(1)
                    Ol = (PQ[rows] @ Ht - A @ V[ks]) / den[:, None]
                    s[rows] = (1 - a) / den
                    dd[rows] = -(1 - a) * (G[rows] * Ol).sum(1) / den
                D[rows] = a * (G[rows] * Os).sum(1)
                dH_i.append(PQ[rows].T @ (s[rows][:, None] * G[rows]))
                dZ_i.append(PQ[rows].T @ dd[rows])
            dHt, dZt = np.sum(dH_i, axis=0), np.sum(dZ_i, axis=0)
            for j in range(nkv):
                ks = keys_of[j]
                users = [i for i in range(nq) if j in set(int(x) for x in kept[b, h, i])]
                M = dHt - sum((dH_i[i] for i in users), np.zeros((d, d)))
                z = dZt - sum((dZ_i[i] for i in users), np.zeros(d))
                dvj = PK[ks] @ M
                dkj = np.zeros((len(ks), d))
                for i in users:
                    rows = np.arange(i * bq, min((i + 1) * bq, N))
                    a = alpha[b, h, i]
                    P = np.exp(sc * Q[rows] @ K[ks].T - lse[rows][:, None])
                    dS = P * (a * (G[rows] @ V[ks].T) - D[rows][:, None])
                    dvj += (a * P).T @ G[rows]
                    dkj += sc * dS.T @ Q[rows]
                dphi = V[ks] @ M.T + z[None, :]
                dv[b, h, ks] = dvj
                dk[b, h, ks] = dkj + _phi_grad(K[ks], dphi, kind)
    return {"dq": base["dq"], "dk": dk, "dv": dv, "dalpha": base["dalpha"]}


@pytest.mark.parametrize("N,d,bq,kk,kind", [(300, 16, 128, 2, "elu1"), (333, 8, 128, 3, "softmax"),
                                            (130, 16, 128, 0, "elu1"), (256, 16, 128, 4, "elu1")])
def test_key_side_from_tile_partials_matches_oracle(N, d, bq, kk, kind):
    rng = np.random.default_rng(13 * N + kk)
    H, bkv = 2, 64
    q, k, v, do = (rng.standard_normal((1, H, N, d)) for _ in range(4))
    nq, nkv = -(-N // bq), -(-N // bkv)
    kk = min(kk, nkv)
    kept = np.array([[[np.sort(rng.choice(nkv, kk, replace=False)) for _ in range(nq)] for _ in range(H)]])
    kept = kept.reshape(1, H, nq, kk)
    alpha = rng.uniform(0.1, 0.9, (1, H, nq))
    ref = orc.sla2_backward(q, k, v, kept, alpha, do, bq, bkv, kind)
    got = _key_block_linear_from_tile_partials(q, k, v, kept, alpha, do, bq, bkv, kind)
    for name in ref:
        assert np.allclose(got[name], ref[name], atol=1e-12, rtol=1e-10), name


def _sla_key_side_from_tile_partials(q, k, v, labels, wp, do, bq, bkv, kind):
    """SLA's backward in the arrangement of the tensor-core SLA2 kernels: per
    query tile i, E_i = dO_i W_proj^T (dO_l), den from the marginal blocks,
    s = 1 / den, dden = -E . O_l / den, dH_i = phi(Q_i)^T (s E_i), dZ_i =
    phi(Q_i)^T dden; per key block j, with L_j the tiles for which j is critical
    or negligible (both leave the linear branch) and C_j those for which it is
    critical (the softmax), M_j = dH_tot - sum over L_j of dH_i:
      dV_j = sum over C_j of P_ij^T dO_i + phi(K_j) M_j
      dphi(K_j) = V_j M_j^T + dZ_tot - sum over L_j of dZ_i
      dK_j = sum over C_j of dS_ij^T Q_i / sqrt(d) + phi'(K_j) dphi(K_j)
    with dS = P * (dO V^T - D), D = dO . O_s; dQ query-major as in SLA2 with E
    for the linear terms; dW_proj = sum O_l^T dO."""
    B, H, N, d = q.shape
    nq, nkv = -(-N // bq), -(-N // bkv)
    sc = 1.0 / math.sqrt(d)
    dq, dk, dv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    dwp = np.zeros(wp.shape)
    for b in range(B):
        for h in range(H):
            Q, K, V, G = q[b, h], k[b, h], v[b, h], do[b, h]
            PK, PQ = _phi(K, kind), _phi(Q, kind)
            Ht, Zt = PK.T @ V, PK.sum(0)
            keys_of = [np.arange(j * bkv, min((j + 1) * bkv, N)) for j in range(nkv)]
            lse, D = np.zeros(N), np.zeros(N)
            dH_i, dZ_i = [], []
            crit_of, out_of = [], []
            for i in range(nq):
                rows = np.arange(i * bq, min((i + 1) * bq, N))
                lab = labels[b, h, i]
                crit = [int(j) for j in np.nonzero(lab == 1)[0]]
                out = [int(j) for j in np.nonzero(lab != 0)[0]]
                crit_of.append(set(crit))
                out_of.append(set(out))
                ks = np.concatenate([keys_of[j] for j in crit]) if crit else np.zeros(0, int)
                ko = np.concatenate([keys_of[j] for j in out]) if out else np.zeros(0, int)
                E = G[rows] @ wp.T
                Os = np.zeros((len(rows), d))
                if len(ks):
                    S = sc * Q[rows] @ K[ks].T
                    mx = S.max(1)
                    lse[rows] = mx + np.log(np.exp(S - mx[:, None]).sum(1))
                    Os = np.exp(S - lse[rows][:, None]) @ V[ks]
                D[rows] = (G[rows] * Os).sum(1)
                s_r, dd_r = np.zeros(len(rows)), np.zeros(len(rows))
                Ol = np.zeros((len(rows), d))
                if len(out) < nkv:
                    A = PQ[rows] @ PK[ko].T if len(ko) else np.zeros((len(rows), 0))
                    den = PQ[rows] @ Zt - A.sum(1)
                    Ol = (PQ[rows] @ Ht - A @ V[ko]) / den[:, None]
                    s_r = 1.0 / den
                    dd_r = -(E * Ol).sum(1) / den
                dwp += Ol.T @ G[rows]
                dH_i.append(PQ[rows].T @ (s_r[:, None] * E))
                dZ_i.append(PQ[rows].T @ dd_r)
                # dQ: the sparse part over the critical blocks, the linear part with E
                dqs = np.zeros((len(rows), d))
                dql = s_r[:, None] * (E @ Ht.T) + dd_r[:, None] * Zt[None, :]
                for j in out:
                    kj = keys_of[j]
                    Bx = s_r[:, None] * (E @ V[kj].T) + dd_r[:, None]
                    dql -= Bx @ PK[kj]
                    if j in crit_of[i]:
                        P = np.exp(sc * Q[rows] @ K[kj].T - lse[rows][:, None])
                        dS = P * (G[rows] @ V[kj].T - D[rows][:, None])
                        dqs += sc * dS @ K[kj]
                dq[b, h, rows] = dqs + _phi_grad(Q[rows], dql, kind)
            dHt, dZt = np.sum(dH_i, axis=0), np.sum(dZ_i, axis=0)
            for j in range(nkv):
                ks = keys_of[j]
                L = [i for i in range(nq) if j in out_of[i]]
                Cr = [i for i in L if j in crit_of[i]]
                M = dHt - sum((dH_i[i] for i in L), np.zeros((d, d)))
                z = dZt - sum((dZ_i[i] for i in L), np.zeros(d))
                dvj = PK[ks] @ M
                dkj = np.zeros((len(ks), d))
                for i in Cr:
                    rows = np.arange(i * bq, min((i + 1) * bq, N))
                    P = np.exp(sc * Q[rows] @ K[ks].T - lse[rows][:, None])
                    dS = P * (G[rows] @ V[ks].T - D[rows][:, None])
                    dvj += P.T @ G[rows]
                    dkj += sc * dS.T @ Q[rows]
                dv[b, h, ks] = dvj
                dk[b, h, ks] = dkj + _phi_grad(K[ks], V[ks] @ M.T + z[None, :], kind)
    return {"dq": dq, "dk": dk, "dv": dv, "dwproj": dwp}


@pytest.mark.parametrize("N,d,bq,kind,n_crit,n_negl", [(300, 16, 128, "elu1", 1, 1), (333, 8, 128, "softmax", 2, 1),
                                                        (130, 16, 128, "elu1", 0, 1), (256, 16, 128, "elu1", 2, 2),
                                                        (256, 16, 128, "elu1", 4, 0)])
def test_sla_key_side_from_tile_partials_matches_oracle(N, d, bq, kind, n_crit, n_negl):
    """The same regrouping for SLA's three labels: critical blocks in the
    softmax, critical and negligible blocks both out of the linear totals,
    dO_l = dO W_proj^T; no critical block, no marginal block, every block
    critical."""
    rng = np.random.default_rng(3 * N + 10 * n_crit + n_negl)
    H, bkv = 2, 64
    q, k, v, do = (rng.standard_normal((1, H, N, d)) for _ in range(4))
    nq, nkv = -(-N // bq), -(-N // bkv)
    labels = np.zeros((1, H, nq, nkv), dtype=np.int8)
    for h, i in np.ndindex(H, nq):
        perm = rng.permutation(nkv)
        labels[0, h, i, perm[:n_crit]] = 1
        labels[0, h, i, perm[n_crit:n_crit + n_negl]] = -1
    wp = rng.standard_normal((d, d)) / math.sqrt(d)
    ref = orc.sla_backward(q, k, v, labels, wp, do, bq, bkv, kind)
    got = _sla_key_side_from_tile_partials(q, k, v, labels, wp, do, bq, bkv, kind)
    for name in ref:
        assert np.allclose(got[name], ref[name], atol=1e-12, rtol=1e-10), name
