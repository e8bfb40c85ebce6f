"""Pins for the CPU oracle: checks against facts fixed by the pages and by
mathematics, each written as a function of the oracle module so that
tests/test_oracle_mutations.py can run them against an oracle with a planted
mistake.  Each raises AssertionError when the pin fails.

Sources: "SLA2 深度解读 …" (jefxiong.cn) §04 (P = P1 + P2, alpha = P1·1,
P1 V = alpha ⊙ (P_s V)), §05 (router, identity projections = SLA heuristic);
"SLA: Beyond Sparsity in Diffusion Transformers …" (papernotes.org) 关键设计 2
(three labels) and 3 (linear branch H_i, Z_i, O_l and O = O_s + Proj(O_l)).
"""
from __future__ import annotations

import math

from fractions import Fraction

import numpy as np
import torch


def _rand(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * scale


# ---------------------------------------------------------------- router pins

def pin_pool_bruteforce(orc):
    """Fixed-order fp32 pooled means equal a scalar loop with np.float32, and
    a ragged last block averages only its own tokens."""
    x = _rand((1, 2, 11, 3), 1).astype(np.float32)
    got = orc.pool_blocks(x, 4)
    assert got.shape == (1, 2, 3, 3)
    for h in range(2):
        for i in range(3):
            toks = range(4 * i, min(4 * i + 4, 11))
            for c in range(3):
                acc = np.float32(0.0)
                for n in toks:
                    acc = np.float32(acc + x[0, h, n, c])
                want = np.float32(acc / np.float32(len(toks)))
                assert got[0, h, i, c] == want, (h, i, c)
    # exact case: small integers
    xi = np.arange(2 * 12, dtype=np.float32).reshape(1, 1, 12, 2)
    gi = orc.pool_blocks(xi, 5)  # blocks of 5, 5, 2 tokens
    assert np.array_equal(gi[0, 0], np.array([[4, 5], [14, 15], [21, 22]], dtype=np.float32))


def _rn32(v: Fraction) -> np.float32:
    """The fp32 nearest to the exact rational v (ties to even), by exact
    comparison with the fp32 neighbours of a first guess."""
    f = np.float32(float(v))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    return min(cands, key=lambda c: (abs(Fraction(float(c)) - v), int(np.float32(c).view(np.uint32)) & 1))


def _fma_chain(xs, ys) -> np.float32:
    """acc = rn32(x * y + acc) over the pairs in order, from +0.0, in exact
    rational arithmetic: each multiply-add rounded once."""
    acc = np.float32(0.0)
    for x, y in zip(xs, ys):
        acc = _rn32(Fraction(float(x)) * Fraction(float(y)) + Fraction(float(acc)))
    return acc


def pin_fma32_exact(orc):
    """The vectorised single-rounding multiply-add equals the exact rational
    result rounded once, on random values and on cancelling ones."""
    g = np.random.default_rng(41)
    a = (g.standard_normal(400) * np.exp2(g.integers(-20, 20, 400))).astype(np.float32)
    b = (g.standard_normal(400) * np.exp2(g.integers(-20, 20, 400))).astype(np.float32)
    c = (g.standard_normal(400) * np.exp2(g.integers(-20, 20, 400))).astype(np.float32)
    c[:100] = -(a[:100].astype(np.float64) * b[:100]).astype(np.float32)  # near-cancelling sums
    got = orc.fma32(a, b, c)
    for i in range(400):
        want = _rn32(Fraction(float(a[i])) * Fraction(float(b[i])) + Fraction(float(c[i])))
        assert got[i] == want, (i, a[i], b[i], c[i], got[i], want)


def pin_fma32_double_rounding_case(orc):
    """A multiply-add where rounding the fp64 sum to fp32 rounds twice and
    goes wrong: a * b = 2^-24 (1 + eta), 0 < eta < 2^-29, plus c = 1.  The fp64
    sum lands exactly on the fp32 midpoint 1 + 2^-24 and ties-to-even would
    give 1; the exact value is above the midpoint, so the answer is 1 + 2^-23."""
    g = np.random.default_rng(7)
    for _ in range(20000):
        a = np.float32(g.uniform(2.0 ** -12, 2.0 ** -11))
        b = np.float32(2.0 ** -24 / float(a))
        eta = Fraction(float(a)) * Fraction(float(b)) / Fraction(1, 2 ** 24) - 1
        if 0 < eta < Fraction(1, 2 ** 29):
            break
    else:
        raise AssertionError("no case found")
    c = np.float32(1.0)
    naive = np.float32(np.float64(a) * np.float64(b) + np.float64(c))
    want = _rn32(Fraction(float(a)) * Fraction(float(b)) + 1)
    assert naive != want and want == np.float32(1.0 + 2.0 ** -23)
    assert orc.fma32(np.array([a]), np.array([b]), np.array([c]))[0] == want


def pin_project_bruteforce(orc):
    """Projection is x W (row vector times matrix), a chain of single-rounding
    multiply-adds in ascending order (checked in exact rational arithmetic);
    W = None and W = I are both the identity; a permutation matrix permutes."""
    x = _rand((1, 1, 3, 4), 2).astype(np.float32)
    w = _rand((4, 4), 3).astype(np.float32)
    got = orc.project(x, w)
    for r in range(3):
        for c in range(4):
            assert got[0, 0, r, c] == _fma_chain(x[0, 0, r, :], w[:, c])
    assert np.array_equal(orc.project(x, None), x)
    assert np.array_equal(orc.project(x, np.eye(4, dtype=np.float32)), x)
    perm = np.eye(4, dtype=np.float32)[[2, 0, 3, 1]]   # x @ perm picks columns
    assert np.array_equal(orc.project(x, perm), x @ perm)
    assert np.allclose(orc.project(x, w), x.astype(np.float64) @ w.astype(np.float64), rtol=1e-5, atol=1e-6)


def pin_scores_bruteforce(orc):
    qt = _rand((1, 1, 3, 5), 4).astype(np.float32)
    kt = _rand((1, 1, 4, 5), 5).astype(np.float32)
    got = orc.block_scores(qt, kt)
    assert got.shape == (1, 1, 3, 4)
    for i in range(3):
        for j in range(4):
            assert got[0, 0, i, j] == _fma_chain(qt[0, 0, i, :], kt[0, 0, j, :])
    ref = qt[0, 0].astype(np.float64) @ kt[0, 0].astype(np.float64).T
    assert np.allclose(got[0, 0], ref, rtol=1e-5, atol=1e-6)


def pin_topk_sort(orc):
    """Top-k equals the first k of a full sort by (score desc, index asc),
    returned ascending; equal scores keep the lower index."""
    s = np.array([[[[0.5, 2.0, 2.0, -1.0, 2.0, 0.5]]]], dtype=np.float32)
    assert orc.topk_blocks(s, 2).tolist() == [[[[1, 2]]]]
    assert orc.topk_blocks(s, 4).tolist() == [[[[0, 1, 2, 4]]]]
    assert orc.topk_blocks(s, 0).shape == (1, 1, 1, 0)
    r = _rand((2, 3, 5, 17), 6).astype(np.float32)
    r[0, 0, 0, 3] = r[0, 0, 0, 9]  # a tie
    for k in (1, 5, 17):
        got = orc.topk_blocks(r, k)
        for idx in np.ndindex(*r.shape[:-1]):
            row = r[idx]
            order = sorted(range(17), key=lambda j: (-float(row[j]), j))
            assert got[idx].tolist() == sorted(order[:k]), (idx, k)


def pin_labels(orc):
    r = _rand((1, 2, 4, 20), 7).astype(np.float32)
    lab = orc.three_way_labels(r, 3, 5)
    assert ((lab == 1).sum(-1) == 3).all() and ((lab == -1).sum(-1) == 5).all()
    for idx in np.ndindex(*r.shape[:-1]):
        row = r[idx]
        order = sorted(range(20), key=lambda j: (-float(row[j]), j))
        assert sorted(np.nonzero(lab[idx] == 1)[0].tolist()) == sorted(order[:3])
        assert sorted(np.nonzero(lab[idx] == -1)[0].tolist()) == sorted(order[-5:])
    # all blocks critical
    assert (orc.three_way_labels(r, 20, 0) == 1).all()


def pin_keep_count(orc):
    assert orc.keep_count(0.03, 512) == 15
    assert orc.keep_count(0.03, 1182) == 35
    assert orc.keep_count(0.05, 512) == 26
    assert orc.keep_count(0.10, 512) == 51
    assert orc.keep_count(0.05, 1182) == 59
    assert orc.keep_count(0.10, 1182) == 118
    assert orc.keep_count(0.0, 512) == 0
    assert orc.keep_count(1e-9, 512) == 1
    assert orc.keep_count(1.0, 512) == 512
    assert orc.keep_count(2.0, 16) == 16
    assert orc.keep_count(0.25, 16) == 4


def pin_router_identity_and_permutation(orc):
    """W = I gives the pooled heuristic of SLA; permuting whole key blocks
    permutes the selected set accordingly."""
    q = _rand((1, 2, 40, 8), 8).astype(np.float32)
    k = _rand((1, 2, 40, 8), 9).astype(np.float32)
    eye = np.eye(8, dtype=np.float32)
    a = orc.route(q, k, None, None, 8, 8, "sla2", 2)
    b = orc.route(q, k, eye, eye, 8, 8, "sla2", 2)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[2], b[2])
    # heuristic equals ranking of pooled dot products computed in fp64
    qb = q.reshape(1, 2, 5, 8, 8).astype(np.float64).mean(3)
    kb = k.reshape(1, 2, 5, 8, 8).astype(np.float64).mean(3)
    s64 = qb @ np.swapaxes(kb, -1, -2)
    want = np.sort(np.argsort(-s64, axis=-1, kind="stable")[..., :2], -1)
    assert np.array_equal(a[0], want)
    # permute key blocks
    perm = np.array([3, 0, 4, 1, 2])
    kp = k.reshape(1, 2, 5, 8, 8)[:, :, perm].reshape(1, 2, 40, 8)
    c = orc.route(q, kp, None, None, 8, 8, "sla2", 2)
    # block j of kp is block perm[j] of k
    assert np.array_equal(np.sort(perm[c[0]], -1), a[0])
    assert np.array_equal(c[2], a[2][..., perm])


# ------------------------------------------------------------- attention pins

def _full_attention_torch(q, k, v):
    qt, kt, vt = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).numpy()


def _tiny(seed, B=1, H=2, N=44, d=8, scale=1.0):
    return (_rand((B, H, N, d), seed, scale), _rand((B, H, N, d), seed + 1, scale),
            _rand((B, H, N, d), seed + 2))


def pin_all_kept_is_full_attention(orc):
    """Pin 1: every block kept and alpha = 1 -> softmax(QK^T/sqrt d) V."""
    q, k, v = _tiny(10)
    bq, bkv = 8, 6
    nq, nkv = -(-44 // bq), -(-44 // bkv)
    kept = np.broadcast_to(np.arange(nkv), (1, 2, nq, nkv))
    out = orc.sla2_forward(q, k, v, kept, np.ones((1, 2, nq)), bq, bkv)
    assert np.allclose(out["o"], _full_attention_torch(q, k, v), atol=1e-12, rtol=1e-12)
    assert np.all(out["o_l"] == 0.0)


def _expanded_mask(kept, N, bq, bkv):
    B, H, nq, _ = kept.shape
    M = np.zeros((B, H, N, N), dtype=bool)
    for b, h, i in np.ndindex(B, H, nq):
        for j in kept[b, h, i]:
            M[b, h, i * bq:min((i + 1) * bq, N), j * bkv:min((j + 1) * bkv, N)] = True
    return M


def pin_masked_mass_identity(orc):
    """Pin 2: with alpha_true = P1·1 per row and the linear part replaced by the
    exact P2 V, alpha_true ⊙ O_s + P2 V = P V (P = P1 + P2, P1 V = alpha ⊙ P_s V)."""
    q, k, v = _tiny(20, scale=1.5)
    N, d, bq, bkv = 44, 8, 8, 6
    nq, nkv = -(-N // bq), -(-N // bkv)
    rng = np.random.default_rng(21)
    kept = np.stack([np.sort(rng.choice(nkv, 3, replace=False)) for _ in range(2 * nq)]).reshape(1, 2, nq, 3)
    out = orc.sla2_forward(q, k, v, kept, np.ones((1, 2, nq)), bq, bkv)
    s = q @ np.swapaxes(k, -1, -2) / math.sqrt(d)
    P = torch.softmax(torch.from_numpy(s), dim=-1).numpy()
    M = _expanded_mask(kept, N, bq, bkv)
    P1, P2 = np.where(M, P, 0.0), np.where(M, 0.0, P)
    alpha_true = P1.sum(-1, keepdims=True)
    lhs = alpha_true * out["o_s"] + P2 @ v
    assert np.allclose(lhs, P @ v, atol=1e-12, rtol=1e-12)


def pin_nothing_kept_is_linear_attention(orc):
    """Pin 3: no block kept and alpha = 0 -> phi(Q)(phi(K)^T V)/(phi(Q)·sum phi(K))
    over all keys, for both feature maps."""
    q, k, v = _tiny(30)
    for kind in ("elu1", "softmax"):
        out = orc.sla2_forward(q, k, v, np.zeros((1, 2, 6, 0), dtype=np.int32), np.zeros((1, 2, 6)), 8, 6, kind)
        if kind == "elu1":
            fq = torch.nn.functional.elu(torch.from_numpy(q)) + 1
            fk = torch.nn.functional.elu(torch.from_numpy(k)) + 1
        else:
            fq = torch.softmax(torch.from_numpy(q), -1)
            fk = torch.softmax(torch.from_numpy(k), -1)
        num = fq @ (fk.transpose(-1, -2) @ torch.from_numpy(v))
        den = fq @ fk.sum(-2, keepdim=True).transpose(-1, -2)
        want = (num / den).numpy()
        assert np.allclose(out["o"], want, atol=1e-12, rtol=1e-12), kind
        assert np.all(out["o_s"] == 0.0)


def _bruteforce(q, k, v, M, alpha_rows, phi_kind, wproj=None, negl=None):
    """Token-level loops over an expanded N x N mask: sparse weights e^{q.k/sqrt d}
    on M, linear weights phi(q).phi(k) on the rest (minus negligible keys)."""
    B, H, N, d = q.shape
    out = np.zeros_like(v)

    def ph(x):
        if phi_kind == "elu1":
            return [xi + 1.0 if xi > 0 else math.exp(xi) for xi in x]
        m = max(x)
        e = [math.exp(xi - m) for xi in x]
        return [ei / sum(e) for ei in e]

    for b in range(B):
        for h in range(H):
            for n in range(N):
                qn = q[b, h, n]
                fs = [(m, math.exp(sum(qn[c] * k[b, h, m, c] for c in range(d)) / math.sqrt(d)))
                      for m in range(N) if M[b, h, n, m]]
                lin = [m for m in range(N) if not M[b, h, n, m] and not (negl is not None and negl[b, h, n, m])]
                os_ = [0.0] * d
                if fs:
                    den = sum(w for _, w in fs)
                    os_ = [sum(w * v[b, h, m, c] for m, w in fs) / den for c in range(d)]
                ol = [0.0] * d
                if lin:
                    fq = ph(qn)
                    ws = [(m, sum(a * bb for a, bb in zip(fq, ph(k[b, h, m])))) for m in lin]
                    den = sum(w for _, w in ws)
                    ol = [sum(w * v[b, h, m, c] for m, w in ws) / den for c in range(d)]
                if wproj is None:
                    a = alpha_rows[b, h, n]
                    out[b, h, n] = [a * os_[c] + (1 - a) * ol[c] for c in range(d)]
                else:
                    out[b, h, n] = [os_[c] + sum(ol[e] * wproj[e, c] for e in range(d)) for c in range(d)]
    return out


def pin_bruteforce_sla2(orc):
    """Pin 4: blocked SLA2 oracle equals token-level loops on a ragged tiny case."""
    N, d, bq, bkv = 10, 3, 4, 3
    q, k, v = _rand((1, 2, N, d), 40), _rand((1, 2, N, d), 41), _rand((1, 2, N, d), 42)
    nq, nkv = 3, 4
    kept = np.array([[[[0, 3], [1, 2], [2, 3]], [[1, 3], [0, 1], [0, 2]]]])
    alpha = np.array([[[0.2, 0.7, 0.9], [0.5, 0.1, 0.6]]])
    M = _expanded_mask(kept, N, bq, bkv)
    arow = np.repeat(alpha, bq, axis=-1)[..., :N]
    for kind in ("elu1", "softmax"):
        got = orc.sla2_forward(q, k, v, kept, alpha, bq, bkv, kind)["o"]
        want = _bruteforce(q, k, v, M, arow, kind)
        assert np.allclose(got, want, atol=1e-12, rtol=1e-12), kind


def pin_bruteforce_sla(orc):
    """Pin 4 (SLA): critical -> softmax, marginal -> linear, negligible skipped,
    O = O_s + O_l W_proj, against token-level loops."""
    N, d, bq, bkv = 10, 3, 4, 3
    q, k, v = _rand((1, 1, N, d), 50), _rand((1, 1, N, d), 51), _rand((1, 1, N, d), 52)
    wp = _rand((d, d), 53)
    labels = np.array([[[[1, -1, 0, 0], [0, 1, -1, 0], [-1, 0, 0, 1]]]], dtype=np.int8)
    crit = np.zeros((1, 1, N, N), bool)
    negl = np.zeros((1, 1, N, N), bool)
    for i in range(3):
        for j in range(4):
            sl = (0, 0, slice(i * bq, min(i * bq + bq, N)), slice(j * bkv, min(j * bkv + bkv, N)))
            crit[sl] = labels[0, 0, i, j] == 1
            negl[sl] = labels[0, 0, i, j] == -1
    got = orc.sla_forward(q, k, v, labels, wp, bq, bkv)["o"]
    want = _bruteforce(q, k, v, crit, None, "elu1", wproj=wp, negl=negl)
    assert np.allclose(got, want, atol=1e-12, rtol=1e-12)


def pin_total_minus_kept(orc):
    """Pin 5: the direct sum over unselected blocks equals (total - kept) of
    the per-block h_j = phi(K_j)^T V_j, z_j = colsum phi(K_j)."""
    q, k, v = _tiny(60)
    N, bq, bkv = 44, 8, 6
    kept = np.array([1, 4, 6])
    rows = np.arange(8, 16)
    keys_kept = np.concatenate([np.arange(j * bkv, min(j * bkv + bkv, N)) for j in kept])
    keys_uns = np.setdiff1d(np.arange(N), keys_kept)
    o_direct = orc.linear_branch(q[0, 0], k[0, 0], v[0, 0], rows, keys_uns)
    fk = orc.phi(k[0, 0])
    H = fk.T @ v[0, 0] - fk[keys_kept].T @ v[0, 0, keys_kept]
    Z = fk.sum(0) - fk[keys_kept].sum(0)
    fq = orc.phi(q[0, 0, rows])
    assert np.allclose(o_direct, (fq @ H) / (fq @ Z)[:, None], rtol=1e-10, atol=1e-12)


def pin_closed_forms(orc):
    """Constant V -> O equals that vector; identical keys -> uniform weights, so
    O_s and O_l are plain means of V over kept / unselected tokens."""
    N, d, bq, bkv = 20, 4, 5, 4
    q = _rand((1, 1, N, d), 70)
    k = _rand((1, 1, N, d), 71)
    u = np.array([0.5, -2.0, 3.0, 0.25])
    v = np.broadcast_to(u, (1, 1, N, d)).copy()
    kept = np.array([[[[0, 2], [1, 4], [3, 4], [0, 1]]]])
    alpha = np.array([[[0.3, 0.6, 0.1, 0.9]]])
    o = orc.sla2_forward(q, k, v, kept, alpha, bq, bkv)["o"]
    assert np.allclose(o, u, atol=1e-12)
    kc = np.broadcast_to(_rand((d,), 72), (1, 1, N, d)).copy()
    vr = _rand((1, 1, N, d), 73)
    out = orc.sla2_forward(q, kc, vr, kept, alpha, bq, bkv)
    for i in range(4):
        rows = slice(i * bq, (i + 1) * bq)
        kt = np.concatenate([np.arange(j * bkv, (j + 1) * bkv) for j in kept[0, 0, i]])
        ut = np.setdiff1d(np.arange(N), kt)
        ms, ml = vr[0, 0, kt].mean(0), vr[0, 0, ut].mean(0)
        assert np.allclose(out["o_s"][0, 0, rows], ms, atol=1e-12)
        assert np.allclose(out["o_l"][0, 0, rows], ml, atol=1e-12)
        assert np.allclose(out["o"][0, 0, rows], alpha[0, 0, i] * ms + (1 - alpha[0, 0, i]) * ml, atol=1e-12)


def pin_sla_special_cases(orc):
    """SLA with W_proj = 0 is block-sparse attention over the critical blocks;
    all blocks critical is full attention."""
    q, k, v = _tiny(80)
    N, bq, bkv = 44, 8, 6
    nq, nkv = 6, 8
    rng = np.random.default_rng(81)
    lab = np.zeros((1, 2, nq, nkv), np.int8)
    for h, i in np.ndindex(2, nq):
        js = rng.permutation(nkv)
        lab[0, h, i, js[:2]] = 1
        lab[0, h, i, js[2:4]] = -1
    o0 = orc.sla_forward(q, k, v, lab, np.zeros((8, 8)), bq, bkv)["o"]
    kept = np.sort(np.argsort(-lab, axis=-1, kind="stable")[..., :2], -1)
    o2 = orc.sla2_forward(q, k, v, kept, np.ones((1, 2, nq)), bq, bkv)["o"]
    assert np.allclose(o0, o2, atol=1e-12)
    allc = np.ones((1, 2, nq, nkv), np.int8)
    of = orc.sla_forward(q, k, v, allc, _rand((8, 8), 82), bq, bkv)["o"]
    assert np.allclose(of, _full_attention_torch(q, k, v), atol=1e-12)


# ---------------------------------------------------------------- fp8 codec

def pin_e4m3_codec(orc):
    """e4m3 encoder/decoder against torch.float8_e4m3fn: every code, every
    midpoint between neighbouring codes, saturation and signed zero."""
    codes = np.arange(256, dtype=np.uint8)
    tvals = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    dec = orc.e4m3_decode(codes)
    fin = ~np.isnan(tvals)
    assert np.array_equal(dec[fin], tvals[fin]) and np.isnan(dec[~fin]).all()
    pos = np.sort(np.unique(tvals[fin & (tvals >= 0)]))
    mids = (pos[:-1] + pos[1:]) / 2
    xs = np.concatenate([pos, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9), [448.0, 449.0, 464.0, 480.0, 1e6, 3e38]])
    xs = np.concatenate([xs, -xs]).astype(np.float32)
    want = torch.from_numpy(np.clip(xs, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = orc.e4m3_encode(xs)
    assert np.array_equal(got, want)
    assert orc.e4m3_encode(np.array([-0.0], np.float32))[0] == 0x80


def pin_hand_example(orc):
    """A 4-token example worked by hand (d = 4, bq = bkv = 2, L = ln 3).

    q0 = (2L,0,0,0), q2 = (0,0,2L,0), q1 = q3 = 0; k0 = e0, k2 = e2, k1 = k3 = 0;
    v_n = e_n.  Pooled router (W = I): Qbar = (L,0,0,0), (0,0,L,0); Kbar = (1/2,0,0,0),
    (0,0,1/2,0), so the top-1 block of query block 0 is key block 0 and of query
    block 1 is key block 1.  Row 0: scores (L, 0) -> softmax weights (3/4, 1/4);
    phi(q0) = (2L+1,1,1,1), phi(k2) = (1,1,2,1), phi(k3) = (1,1,1,1) -> linear
    weights (2L+5, 2L+4).  Row 1: q = 0 -> uniform softmax (1/2, 1/2) and linear
    weights (5, 4).  Rows 2, 3 mirror rows 0, 1 with the blocks swapped."""
    L = math.log(3.0)
    q = np.zeros((1, 1, 4, 4))
    k = np.zeros((1, 1, 4, 4))
    q[0, 0, 0, 0] = 2 * L
    q[0, 0, 2, 2] = 2 * L
    k[0, 0, 0, 0] = 1.0
    k[0, 0, 2, 2] = 1.0
    v = np.eye(4).reshape(1, 1, 4, 4)
    kept, _, _ = orc.route(q.astype(np.float32), k.astype(np.float32), None, None, 2, 2, "sla2", 1)
    assert kept.tolist() == [[[[0], [1]]]]
    alpha = np.array([[[0.25, 0.5]]])
    o = orc.sla2_forward(q, k, v, kept, alpha, 2, 2)["o"][0, 0]
    w = 4 * L + 9
    want = np.array([
        0.25 * np.array([3 / 4, 1 / 4, 0, 0]) + 0.75 * np.array([0, 0, (2 * L + 5) / w, (2 * L + 4) / w]),
        0.25 * np.array([1 / 2, 1 / 2, 0, 0]) + 0.75 * np.array([0, 0, 5 / 9, 4 / 9]),
        0.5 * np.array([0, 0, 3 / 4, 1 / 4]) + 0.5 * np.array([(2 * L + 5) / w, (2 * L + 4) / w, 0, 0]),
        0.5 * np.array([0, 0, 1 / 2, 1 / 2]) + 0.5 * np.array([5 / 9, 4 / 9, 0, 0]),
    ])
    assert np.allclose(o, want, atol=1e-14, rtol=0)


# ---------------------------------------------------------------- fp8 branch

def _fp8_case(seed, N=300, d=16, offset=0.0):
    q, k, v = _rand((1, 1, N, d), seed), _rand((1, 1, N, d), seed + 1) + offset, _rand((1, 1, N, d), seed + 2)
    kept = np.array([[[[0, 2], [1, 3], [0, 4]]]])
    alpha = np.array([[[0.3, 0.6, 0.9]]])
    return q, k, v, kept, alpha


def pin_fp8_identity_codec_is_fp64(orc):
    """With the e4m3 round trip replaced by the identity, the low-bit branch's
    bookkeeping (smoothing, per-block and per-channel scales, online softmax,
    P scaling) must give the fp64 SLA2 output up to fp32 rounding of K' and of
    the scaled values."""
    q, k, v, kept, alpha = _fp8_case(90)
    ident = lambda x: np.asarray(x, np.float64)  # noqa: E731
    a = orc.sla2_forward(q, k, v, kept, alpha, 128, 64)["o"]
    b = orc.sla2_forward_fp8(q, k, v, kept, alpha, 128, 64, codec=ident)["o"]
    assert np.abs(a - b).max() < 1e-6


def pin_fp8_quantisation_error_bounded(orc):
    """e4m3 keeps 3 mantissa bits: the output moves, but by a bounded amount."""
    q, k, v, kept, alpha = _fp8_case(91)
    a = orc.sla2_forward(q, k, v, kept, alpha, 128, 64)["o"]
    c = orc.sla2_forward_fp8(q, k, v, kept, alpha, 128, 64)["o"]
    err = np.abs(a - c).max()
    assert 1e-4 < err < 0.2, err


def pin_fp8_k_smoothing(orc):
    """A constant offset on every key row does not change softmax attention;
    after K smoothing it does not change the quantised branch either (the mean
    is removed before quantising).  Without smoothing the offset would swamp
    the e4m3 scale."""
    q, k, v, kept, alpha = _fp8_case(92)
    k_off = k + 40.0
    # the linear branch does see the offset: compare the sparse part only
    a = orc.sla2_forward_fp8(q, k, v, kept, alpha, 128, 64)["o_s"]
    b = orc.sla2_forward_fp8(q, k_off, v, kept, alpha, 128, 64)["o_s"]
    assert np.abs(a - b).max() < 0.02


def pin_fp8_block_scales(orc):
    """Per-block scale = amax/448 and codes of x*448/amax: a block whose amax
    is 448 quantises representable values exactly."""
    x = np.array([[448.0, -2.0], [0.5, 3.0], [1.0, 0.0]], dtype=np.float32)
    vals, scales = orc._quant_blocks(x, 2, orc.e4m3_round)
    assert np.allclose(scales, [1.0, 1.0 / 448.0])
    assert np.array_equal(vals[:2], np.array([[448.0, -2.0], [0.5, 3.0]]))
    assert np.array_equal(vals[2], [448.0, 0.0]) and np.allclose(vals[2] * scales[1], [1.0, 0.0])


def pin_fp8_tile_width_exact_without_quantisation(orc):
    """Online softmax is exact for any grouping of the kept blocks into tiles:
    with the identity codec, tiles of 1, 2 or 3 kept blocks (3 kept per row,
    so the grouping 2 + 1 occurs) agree up to the fp32 rounding of p * 448,
    and match the fp64 SLA2 output."""
    q, k, v, _, alpha = _fp8_case(93)
    kept = np.array([[[[0, 2, 4], [1, 3, 4], [0, 1, 2]]]])
    ident = lambda x: np.asarray(x, np.float64)  # noqa: E731
    outs = [orc.sla2_forward_fp8(q, k, v, kept, alpha, 128, 64, codec=ident, kv_tile=t)["o"] for t in (1, 2, 3)]
    # the values reaching the codec are still rounded to fp32 against each tile's max
    assert max(np.abs(outs[0] - o).max() for o in outs[1:]) < 1e-6
    ref = orc.sla2_forward(q, k, v, kept, alpha, 128, 64)["o"]
    assert np.abs(outs[1] - ref).max() < 1e-6


def pin_fp8_tile_width_moves_quantisation(orc):
    """With e4m3 on, P is quantised against the running max of its tile, so
    the tile width changes the rounding (and only the rounding): the outputs
    for 1 and 3 blocks per tile differ, by no more than the quantisation
    error itself."""
    q, k, v, _, alpha = _fp8_case(94)
    kept = np.array([[[[0, 2, 4], [1, 3, 4], [0, 1, 2]]]])
    a = orc.sla2_forward_fp8(q, k, v, kept, alpha, 128, 64, kv_tile=1)["o_s"]
    b = orc.sla2_forward_fp8(q, k, v, kept, alpha, 128, 64, kv_tile=3)["o_s"]
    d = np.abs(a - b).max()
    assert 0.0 < d < 0.1, d


# ---------------------------------------------------------------- SoftTop-k pins
# "SLA2 深度解读 …" (jefxiong.cn) §06 Stage 1: SoftTop-k(P_c)_ij = sigmoid(P_c_ij / tau
# + lambda_i), tau = 0.1, lambda_i by bisection so the row's soft selections sum to
# the budget.

def pin_soft_topk_two_blocks_closed_form(orc):
    """n = 2, k = 1: sigmoid(a + l) + sigmoid(b + l) = 1 has the root
    l = -(a + b) / 2 (as sigmoid(u) + sigmoid(-u) = 1), so the mask is
    [1 / (1 + e^{-(a-b)/2}), 1 / (1 + e^{(a-b)/2})] with a, b = s / tau."""
    for s0, s1, tau in ((0.3, -0.2, 0.1), (1.5, 1.4, 0.1), (-2.0, 0.7, 0.5)):
        m, lam = orc.soft_topk(np.array([[s0, s1]]), 1, tau=tau)
        a, b = s0 / tau, s1 / tau
        want = [1.0 / (1.0 + math.exp(-(a - b) / 2)), 1.0 / (1.0 + math.exp((a - b) / 2))]
        assert np.allclose(m[0], want, rtol=0, atol=1e-12), (m, want)
        assert abs(lam[0] + (a + b) / 2) < 1e-9, (lam, a, b)


def pin_soft_topk_equal_scores(orc):
    """All scores equal: by symmetry every block gets k / n, and
    lambda = log(k / (n - k)) - s / tau."""
    for n, k, sv in ((512, 15, 0.37), (16, 4, -1.2), (7, 6, 0.0)):
        m, lam = orc.soft_topk(np.full((2, n), sv), k)
        assert np.allclose(m, k / n, rtol=0, atol=1e-12), m[0, :3]
        assert np.allclose(lam, math.log(k / (n - k)) - sv / 0.1, rtol=0, atol=1e-9), lam


def pin_soft_topk_budget_and_order(orc):
    """Random rows: the soft selections sum to k, lie in (0, 1) and keep the
    order of the scores."""
    s = _rand((6, 200), 301, scale=0.4)
    for k in (1, 6, 50, 199):
        m, _ = orc.soft_topk(s, k)
        assert np.allclose(m.sum(axis=-1), k, rtol=0, atol=1e-9), m.sum(axis=-1)
        assert (m > 0).all() and (m < 1).all()
        for r in range(s.shape[0]):
            o = np.argsort(s[r])
            assert (np.diff(m[r][o]) >= 0).all()


def pin_soft_topk_hard_limit(orc):
    """As tau -> 0 the soft mask becomes the hard Top-k: rows whose k best
    scores are >= 1 and the rest <= 0 give ~1 on the hard Top-k set and ~0
    elsewhere at tau = 1e-3."""
    g = np.random.default_rng(302)
    n, k = 40, 7
    s = np.empty((5, n))
    for r in range(5):
        idx = g.permutation(n)
        s[r, idx[:k]] = 1.0 + g.random(k)
        s[r, idx[k:]] = -g.random(n - k)
    m, _ = orc.soft_topk(s, k, tau=1e-3)
    hard = np.zeros((5, n))
    np.put_along_axis(hard, orc.topk_blocks(s, k).astype(np.int64), 1.0, axis=-1)
    assert np.abs(m - hard).max() < 1e-6, np.abs(m - hard).max()


def pin_soft_topk_edges_and_shift(orc):
    """k = 0 selects nothing, k = n everything; adding c to a row leaves the
    mask unchanged and moves lambda by -c / tau."""
    s = _rand((3, 30), 303)
    m0, l0 = orc.soft_topk(s, 0)
    mn, ln = orc.soft_topk(s, 30)
    assert (m0 == 0).all() and np.isneginf(l0).all()
    assert (mn == 1).all() and np.isposinf(ln).all()
    m, lam = orc.soft_topk(s, 9)
    m2, lam2 = orc.soft_topk(s + 2.5, 9)
    assert np.allclose(m, m2, rtol=0, atol=1e-10)
    assert np.allclose(lam2, lam - 25.0, rtol=0, atol=1e-8)


# ---------------------------------------------------------------- INT8 variant pins

def pin_int8_codec(orc):
    """INT8 round trip: round to nearest with ties to even (as torch.round),
    saturated to [-127, 127]."""
    x = np.array([2.5, 3.5, -2.5, -3.5, 0.49, 126.6, 127.4, 200.0, -300.0, -127.5, 0.0], dtype=np.float32)
    want = np.array([2, 4, -2, -4, 0, 127, 127, 127, -127, -127, 0], dtype=np.float64)
    assert np.array_equal(orc.int8_round(x), want)
    g = _rand((4000,), 95, 80.0).astype(np.float32)
    ref = torch.clamp(torch.round(torch.from_numpy(g).double()), -127, 127).numpy()
    assert np.array_equal(orc.int8_round(g), ref)


def pin_int8_integer_inputs_are_exact(orc):
    """Q and K' integer-valued with |x| <= 127 and 127 reached in every 128-token
    block: the INT8 codes are the values themselves, so with P and V left
    unquantised the INT8 branch equals the fp64 sparse branch.  e4m3 cannot
    hold these integers (3 mantissa bits), so the same case through e4m3 Q, K'
    does move."""
    g = np.random.default_rng(96)
    N, d = 256, 16
    q = g.integers(-127, 128, size=(1, 1, N, d)).astype(np.float64)
    blocks = []
    for blk in range(2):
        q[0, 0, 128 * blk, 0] = 127.0
        half = g.integers(-127, 128, size=(64, d)).astype(np.float64)
        half[0, 1] = 127.0
        blocks += [half, -half]  # every column of every block sums to zero
    kp = np.concatenate(blocks)
    k = (kp + 3.0)[None, None]  # column mean exactly 3, so K' = kp
    v = _rand((1, 1, N, d), 97)
    kept = np.array([[[[0, 2], [1, 3]]]])
    alpha = np.array([[[0.5, 0.5]]])
    ident = lambda x: np.asarray(x, np.float64)  # noqa: E731
    sq, sk = q * 2.0 ** -6, k * 2.0 ** -6  # exact: amax 127/64, inv 64, scale 1/64
    # P and V pass through fp32 on every path; only the Q, K' round trip differs
    a = orc.sla2_forward_fp8(sq, sk, v, kept, alpha, 128, 64, codec=ident, qk_codec=ident, qk_max=127.0)["o_s"]
    b = orc.sla2_forward_fp8(sq, sk, v, kept, alpha, 128, 64, codec=ident,
                             qk_codec=orc.int8_round, qk_max=127.0)["o_s"]
    assert np.abs(a - b).max() < 1e-12
    assert np.abs(a - orc.sla2_forward(sq, sk, v, kept, alpha, 128, 64)["o_s"]).max() < 1e-6
    c = orc.sla2_forward_fp8(sq, sk, v, kept, alpha, 128, 64, codec=ident,
                             qk_codec=orc.e4m3_round, qk_max=448.0)["o_s"]
    assert np.abs(a - c).max() > 1e-4


def pin_int8_variant_error_bounded(orc):
    """The INT8 variant (INT8 Q, K'; e4m3 P, V) moves the output by a bounded
    amount, and its scale bookkeeping with qmax 127 is exact when every round
    trip is the identity."""
    q, k, v, kept, alpha = _fp8_case(98)
    a = orc.sla2_forward(q, k, v, kept, alpha, 128, 64)["o"]
    c = orc.sla2_forward_int8(q, k, v, kept, alpha, 128, 64)["o"]
    err = np.abs(a - c).max()
    assert 1e-4 < err < 0.2, err
    ident = lambda x: np.asarray(x, np.float64)  # noqa: E731
    b = orc.sla2_forward_fp8(q, k, v, kept, alpha, 128, 64, codec=ident, qk_codec=ident, qk_max=127.0)["o"]
    assert np.abs(a - b).max() < 1e-6


# ---------------------------------------------------------------- backward pins
# The backward is pinned by central finite differences of the (pinned) forward,
# by torch autograd on the two limits that are textbook attention, and by sum
# rules that follow from the forward's structure.

def _bwd_case(seed, N=45, d=8, H=2, bq=16, bkv=8, k_keep=2):
    g = np.random.default_rng(seed)
    q = g.standard_normal((1, H, N, d)) * 0.8
    k = g.standard_normal((1, H, N, d)) * 0.8
    v = g.standard_normal((1, H, N, d))
    nq, nkv = -(-N // bq), -(-N // bkv)
    kept = np.array([[[np.sort(g.choice(nkv, k_keep, replace=False)) for _ in range(nq)] for _ in range(H)]])
    alpha = g.uniform(0.15, 0.85, (1, H, nq))
    do = g.standard_normal((1, H, N, d))
    return q, k, v, kept, alpha, do


def _fd_agree(loss, x, grad, n, seed, h=1e-5, tol=1e-6):
    """Central differences of loss at n sampled entries of x against grad."""
    idx = np.random.default_rng(seed).choice(x.size, size=min(n, x.size), replace=False)
    for t in idx:
        xp, xm = x.copy(), x.copy()
        xp.flat[t] += h
        xm.flat[t] -= h
        fd = (loss(xp) - loss(xm)) / (2.0 * h)
        assert abs(fd - grad.flat[t]) <= tol * (1.0 + abs(fd)), (int(t), fd, float(grad.flat[t]))


def _sla2_fd(orc, kind, seed, n):
    q, k, v, kept, alpha, do = _bwd_case(seed)
    bq, bkv = 16, 8
    gr = orc.sla2_backward(q, k, v, kept, alpha, do, bq, bkv, kind)

    def L(q_=q, k_=k, v_=v, a_=alpha):
        return float((orc.sla2_forward(q_, k_, v_, kept, a_, bq, bkv, kind)["o"] * do).sum())
    _fd_agree(lambda x: L(q_=x), q, gr["dq"], n, seed + 1)
    _fd_agree(lambda x: L(k_=x), k, gr["dk"], n, seed + 2)
    _fd_agree(lambda x: L(v_=x), v, gr["dv"], n, seed + 3)
    _fd_agree(lambda x: L(a_=x), alpha, gr["dalpha"], alpha.size, seed + 4)


def pin_bwd_sla2_finite_differences(orc):
    """SLA2 gradients (dQ, dK, dV, dalpha) against central differences of the
    forward, ELU+1 feature map, ragged last blocks."""
    _sla2_fd(orc, "elu1", 700, 24)


def pin_bwd_sla2_softmax_phi_finite_differences(orc):
    """The same with the softmax feature map."""
    _sla2_fd(orc, "softmax", 710, 16)


def pin_bwd_sla_finite_differences(orc):
    """SLA gradients (dQ, dK, dV, dW_proj) against central differences, with
    critical, marginal and negligible blocks in every row."""
    q, k, v, _, _, do = _bwd_case(720)
    bq, bkv, nq, nkv = 16, 8, 3, 6
    g = np.random.default_rng(721)
    labels = np.zeros((1, 2, nq, nkv), dtype=np.int8)
    for h, i in np.ndindex(2, nq):
        perm = g.permutation(nkv)
        labels[0, h, i, perm[:2]] = 1
        labels[0, h, i, perm[2:3]] = -1
    wp = g.standard_normal((8, 8)) / math.sqrt(8)
    gr = orc.sla_backward(q, k, v, labels, wp, do, bq, bkv)

    def L(q_=q, k_=k, v_=v, w_=wp):
        return float((orc.sla_forward(q_, k_, v_, labels, w_, bq, bkv)["o"] * do).sum())
    _fd_agree(lambda x: L(q_=x), q, gr["dq"], 20, 722)
    _fd_agree(lambda x: L(k_=x), k, gr["dk"], 20, 723)
    _fd_agree(lambda x: L(v_=x), v, gr["dv"], 20, 724)
    _fd_agree(lambda x: L(w_=x), wp, gr["dwproj"], 20, 725)


def pin_bwd_textbook_limits(orc):
    """Every block kept with alpha = 1 is softmax attention, no block kept with
    alpha = 0 is linear attention: their gradients equal torch autograd of
    those textbook formulas (float64)."""
    q, k, v, _, _, do = _bwd_case(730)
    N, bq, bkv, nq, nkv = 45, 16, 8, 3, 6
    tq, tk, tv = (torch.from_numpy(x.copy()).requires_grad_(True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    o.backward(torch.from_numpy(do))
    kept = np.broadcast_to(np.arange(nkv), (1, 2, nq, nkv))
    gr = orc.sla2_backward(q, k, v, kept, np.ones((1, 2, nq)), do, bq, bkv)
    for name, t in (("dq", tq), ("dk", tk), ("dv", tv)):
        assert np.allclose(gr[name], t.grad.numpy(), atol=1e-12, rtol=1e-10), name
    for kind in ("elu1", "softmax"):
        tq, tk, tv = (torch.from_numpy(x.copy()).requires_grad_(True) for x in (q, k, v))
        if kind == "elu1":
            fq, fk = torch.nn.functional.elu(tq) + 1, torch.nn.functional.elu(tk) + 1
        else:
            fq, fk = torch.softmax(tq, -1), torch.softmax(tk, -1)
        o = (fq @ (fk.transpose(-1, -2) @ tv)) / (fq @ fk.sum(-2, keepdim=True).transpose(-1, -2))
        o.backward(torch.from_numpy(do))
        gr = orc.sla2_backward(q, k, v, np.zeros((1, 2, nq, 0), dtype=np.int32), np.zeros((1, 2, nq)), do,
                               bq, bkv, kind)
        for name, t in (("dq", tq), ("dk", tk), ("dv", tv)):
            assert np.allclose(gr[name], t.grad.numpy(), atol=1e-12, rtol=1e-10), (kind, name)


def pin_bwd_sum_rules(orc):
    """Rules that follow from the forward's structure:
    - both branches weight the values convexly, so with 0 < k < n_kv the value
      gradients of a head sum to the sum of its upstream gradients;
    - with alpha = 1 only the softmax acts, and a common shift of the keys
      leaves it unchanged, so the key gradients of a head sum to zero;
    - the softmax feature map ignores a common shift of a token's channels, so
      with alpha = 0 every row of dQ and of dK sums to zero."""
    q, k, v, kept, alpha, do = _bwd_case(740)
    gr = orc.sla2_backward(q, k, v, kept, alpha, do, 16, 8)
    assert np.allclose(gr["dv"].sum(axis=2), do.sum(axis=2), atol=1e-10)
    gr = orc.sla2_backward(q, k, v, kept, np.ones_like(alpha), do, 16, 8)
    assert np.allclose(gr["dk"].sum(axis=2), 0.0, atol=1e-10)
    assert np.abs(gr["dk"]).max() > 1e-3
    gr = orc.sla2_backward(q, k, v, kept, np.zeros_like(alpha), do, 16, 8, "softmax")
    assert np.allclose(gr["dq"].sum(axis=3), 0.0, atol=1e-10)
    assert np.allclose(gr["dk"].sum(axis=3), 0.0, atol=1e-10)
    assert np.abs(gr["dq"]).max() > 1e-3 and np.abs(gr["dk"]).max() > 1e-3
    # the shares of single query blocks add up to the whole gradient
    full = orc.sla2_backward(q, k, v, kept, alpha, do, 16, 8)
    parts = [orc.sla2_backward(q, k, v, kept, alpha, do, 16, 8, blocks=[t]) for t in np.ndindex(1, 2, 3)]
    for name in ("dq", "dk", "dv", "dalpha"):
        assert np.allclose(sum(p[name] for p in parts), full[name], atol=1e-12), name


ALL_PINS = [pin_hand_example, pin_fma32_exact, pin_fma32_double_rounding_case, pin_fp8_identity_codec_is_fp64, pin_fp8_quantisation_error_bounded,
            pin_fp8_k_smoothing, pin_fp8_block_scales, pin_fp8_tile_width_exact_without_quantisation,
            pin_fp8_tile_width_moves_quantisation,
    pin_pool_bruteforce, pin_project_bruteforce, pin_scores_bruteforce, pin_topk_sort,
    pin_labels, pin_keep_count, pin_router_identity_and_permutation,
    pin_all_kept_is_full_attention, pin_masked_mass_identity, pin_nothing_kept_is_linear_attention,
    pin_bruteforce_sla2, pin_bruteforce_sla, pin_total_minus_kept, pin_closed_forms,
    pin_sla_special_cases, pin_e4m3_codec,
    pin_soft_topk_two_blocks_closed_form, pin_soft_topk_equal_scores, pin_soft_topk_budget_and_order,
    pin_soft_topk_hard_limit, pin_soft_topk_edges_and_shift,
    pin_bwd_sla2_finite_differences, pin_bwd_sla2_softmax_phi_finite_differences, pin_bwd_sla_finite_differences,
    pin_bwd_textbook_limits, pin_bwd_sum_rules,
    pin_int8_codec, pin_int8_integer_inputs_are_exact, pin_int8_variant_error_bounded,
]
