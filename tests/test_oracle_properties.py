"""Property tests of the CPU oracle (random shapes and values, on the CPU):
invariants the method fixes at any size, beside the fixed pins.

"SLA2 深度解读 …" (jefxiong.cn) §04 (O = alpha O_s + (1 - alpha) O_l), §05
(hard Top-k of the router map), §06 (SoftTop-k); "SLA: Beyond Sparsity …"
(papernotes.org) 关键设计 2 (three labels).
"""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import sla_oracle as orc

SETTINGS = dict(max_examples=25, deadline=None)


@settings(**SETTINGS)
@given(st.integers(1, 40), st.integers(0, 40), st.integers(0, 2 ** 31 - 1))
def test_topk_is_invariant_under_increasing_maps(n, k, seed):
    """A hard top-k depends only on the order of the scores: an increasing map
    (here x -> 3 x^3 + x - 5, kept in fp32 order) selects the same blocks, and
    the result is ascending, distinct and of size min(k, n)."""
    k = min(k, n)
    g = np.random.default_rng(seed)
    s = g.standard_normal((1, 1, 3, n)).astype(np.float32)
    s[0, 0, 1] = np.round(s[0, 0, 1])  # many ties
    # strictly increasing, and evaluated in fp64 it keeps fp32 ties tied and the
    # order of distinct fp32 values strict, so the same blocks must win
    t = 3.0 * s.astype(np.float64) ** 3 + s - 5.0
    a = orc.topk_blocks(s, k)
    assert a.shape == (1, 1, 3, k)
    for r in range(3):
        row = a[0, 0, r]
        assert list(row) == sorted(set(row.tolist()))
    assert np.array_equal(a, orc.topk_blocks(t, k))


@settings(**SETTINGS)
@given(st.integers(1, 30), st.integers(0, 30), st.integers(0, 30), st.integers(0, 2 ** 31 - 1))
def test_three_labels_partition_each_row(n, kh, kl, seed):
    """Critical and negligible counts are exact, disjoint, and every critical
    score is >= every marginal score >= every negligible score."""
    kh = min(kh, n)
    kl = min(kl, n - kh)
    g = np.random.default_rng(seed)
    s = g.standard_normal((1, 2, 2, n)).astype(np.float32)
    lab = orc.three_way_labels(s, kh, kl)
    for idx in np.ndindex(1, 2, 2):
        row, lr = s[idx], lab[idx]
        assert (lr == 1).sum() == kh and (lr == -1).sum() == kl
        crit, marg, negl = row[lr == 1], row[lr == 0], row[lr == -1]
        if len(crit) and len(marg):
            assert crit.min() >= marg.max()
        if len(marg) and len(negl):
            assert marg.min() >= negl.max()
        if len(crit) and len(negl):
            assert crit.min() >= negl.max()


@settings(**SETTINGS)
@given(st.integers(1, 90), st.sampled_from([8, 16]), st.integers(0, 3), st.floats(0.0, 1.0),
       st.integers(0, 2 ** 31 - 1))
def test_sla2_output_is_affine_in_alpha(N, d, kk, a, seed):
    """O = alpha O_s + (1 - alpha) O_l: the output at any alpha is the mix of
    the outputs at alpha = 1 and alpha = 0."""
    g = np.random.default_rng(seed)
    bq, bkv = 32, 16
    nq, nkv = -(-N // bq), -(-N // bkv)
    kk = min(kk, nkv)
    q, k, v = (g.standard_normal((1, 1, N, d)) for _ in range(3))
    kept = np.array([[[np.sort(g.choice(nkv, kk, replace=False)) for _ in range(nq)]]]).reshape(1, 1, nq, kk)
    one, zero = np.ones((1, 1, nq)), np.zeros((1, 1, nq))
    o1 = orc.sla2_forward(q, k, v, kept, one, bq, bkv)["o"]
    o0 = orc.sla2_forward(q, k, v, kept, zero, bq, bkv)["o"]
    oa = orc.sla2_forward(q, k, v, kept, np.full((1, 1, nq), a), bq, bkv)["o"]
    assert np.allclose(oa, a * o1 + (1 - a) * o0, atol=1e-12)


@settings(**SETTINGS)
@given(st.integers(2, 60), st.integers(1, 59), st.floats(0.02, 2.0), st.integers(0, 2 ** 31 - 1))
def test_soft_topk_budget_and_range(n, k, tau, seed):
    """SoftTop-k entries lie in (0, 1), sum to k per row, and preserve the
    order of the scores."""
    k = min(k, n - 1)
    g = np.random.default_rng(seed)
    s = g.standard_normal((1, 1, 2, n)) * 2.0
    m, lam = orc.soft_topk(s, k, tau=tau)
    assert np.all(m >= 0.0) and np.all(m <= 1.0)
    assert np.allclose(m.sum(-1), k, atol=1e-8)
    for idx in np.ndindex(1, 1, 2):
        o = np.argsort(s[idx])
        assert np.all(np.diff(m[idx][o]) >= -1e-12)


def test_backward_block_shares_add_up():
    """The backward's blocks= option (the oracle computing the share of some
    query blocks only, as the full-size GPU checks use it) splits the gradients
    exactly: the shares of disjoint block sets add up to the full result, for
    SLA2 and SLA."""
    g = np.random.default_rng(41)
    B, H, N, d, bq, bkv = 1, 2, 300, 8, 64, 64
    q, k, v, do = (g.standard_normal((B, H, N, d)) for _ in range(4))
    nq, nkv = -(-N // bq), -(-N // bkv)
    kept = np.stack([np.sort(g.choice(nkv, 2, replace=False)) for _ in range(H * nq)]).reshape(B, H, nq, 2)
    alpha = g.uniform(0.1, 0.9, (B, H, nq))
    labels = np.zeros((B, H, nq, nkv), dtype=np.int8)
    for h, i in np.ndindex(H, nq):
        perm = g.permutation(nkv)
        labels[0, h, i, perm[:1]] = 1
        labels[0, h, i, perm[1:2]] = -1
    wp = g.standard_normal((d, d)) / np.sqrt(d)
    all_blocks = [(0, h, i) for h in range(H) for i in range(nq)]
    first, rest = all_blocks[::2], all_blocks[1::2]
    full = orc.sla2_backward(q, k, v, kept, alpha, do, bq, bkv)
    a = orc.sla2_backward(q, k, v, kept, alpha, do, bq, bkv, blocks=first)
    b = orc.sla2_backward(q, k, v, kept, alpha, do, bq, bkv, blocks=rest)
    for name in full:
        assert np.allclose(a[name] + b[name], full[name], atol=1e-12), name
    full = orc.sla_backward(q, k, v, labels, wp, do, bq, bkv)
    a = orc.sla_backward(q, k, v, labels, wp, do, bq, bkv, blocks=first)
    b = orc.sla_backward(q, k, v, labels, wp, do, bq, bkv, blocks=rest)
    for name in full:
        assert np.allclose(a[name] + b[name], full[name], atol=1e-12), name
