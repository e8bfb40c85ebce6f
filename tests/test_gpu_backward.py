"""GPU parity of sla2_attn_bwd and sla_attn_bwd (the gradients of the SLA2
and SLA forwards with the block mask held fixed) against the oracle's
sla2_backward / sla_backward on the same seeded inputs, element by element.

Follows "SLA: Beyond Sparsity in Diffusion Transformers …" (papernotes.org)
关键设计 4 and "SLA2 深度解读 …" (jefxiong.cn) §07.  The oracle is fp64.

Two paths, two bounds, both relative to each tensor's largest entry:
- the CUDA-core kernels (every shape but the one below) compute in fp32 on
  the exact input values: TOL_BWD_REL, orders of magnitude above fp32
  rounding over a few thousand terms and the order of the atomic adds;
- the tensor-core kernels (bf16 inputs, d = 128, b_q = 128) round dS and
  alpha P - s A to bf16 (unit roundoff 2^-9 = 2e-3) and -Bx sigma, phi(Q)
  to fp16 before the products, on top of the forward's fp16 P in the row
  statistics.  Each output is a sum of such rounded terms, so its error
  relative to the largest entry is about the bf16 unit roundoff: 1.5-3.4e-3
  measured at ragged shapes and at the 1.3B shape.  TOL_BWD_TC bounds the
  largest entry-wise error, TOL_BWD_TC_L2 the relative 2-norm of the error.
"""
import numpy as np
import pytest
import torch

from oracle import sla_oracle as orc
from sparse_linear_attention_b200 import inputs, sla

pytestmark = pytest.mark.gpu

TOL_BWD_REL = 1e-4
TOL_BWD_TC = 1e-2
TOL_BWD_TC_L2 = 5e-3


def _tensor_core(q, bq):
    return q.dtype == torch.bfloat16 and q.shape[-1] == 128 and bq == 128


def _close(name, g, r, tc):
    assert np.isfinite(g).all(), name
    scale = max(np.abs(r).max(), 1e-30)
    err = np.abs(g - r).max() / scale
    assert err <= (TOL_BWD_TC if tc else TOL_BWD_REL), (name, err)
    if tc:
        l2 = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
        assert l2 <= TOL_BWD_TC_L2, (name, l2)


def _kept(seed, B, H, nq, nkv, kk):
    g = np.random.default_rng(seed)
    out = np.zeros((B, H, nq, kk), dtype=np.int32)
    for idx in np.ndindex(B, H, nq):
        out[idx] = np.sort(g.choice(nkv, kk, replace=False))
    return out


def _case(seed, B, H, N, d, bq, kk, dtype):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, H, N, d, generator=g) * 0.8).to(dtype)
    k = (torch.randn(B, H, N, d, generator=g) * 0.8).to(dtype)
    v = torch.randn(B, H, N, d, generator=g).to(dtype)
    do = torch.randn(B, H, N, d, generator=g).to(dtype)
    nq, nkv = -(-N // bq), -(-N // 64)
    alpha = torch.rand(B, H, nq, generator=g) * 0.8 + 0.1
    return q, k, v, do, alpha, _kept(seed, B, H, nq, nkv, kk)


def _run(q, k, v, kept, alpha, do, bq, phi):
    dev = "cuda"
    qd, kd, vd, dod = (t.to(dev).contiguous() for t in (q, k, v, do))
    shape = sla.make_shape(qd, bq, 64)
    B, H, N, d = q.shape
    nq = -(-N // bq)
    kk = kept.shape[-1]
    keptd = torch.from_numpy(kept).to(dev).contiguous() if kk else None
    ws = torch.zeros(sla.sla2_attn_bwd_workspace_size(shape), dtype=torch.uint8, device=dev)
    dq = torch.full((B, H, N, d), float("nan"), device=dev)
    dk = torch.full_like(dq, float("nan"))
    dv = torch.full_like(dq, float("nan"))
    dal = torch.full((B, H, nq), float("nan"), device=dev)
    sla.sla2_attn_bwd(shape, qd, kd, vd, keptd, kk, alpha.to(dev).contiguous(), phi, dod, dq, dk, dv, dal, ws)
    status = sla.sla_read_device_status(ws)
    return status, {"dq": dq.cpu().numpy(), "dk": dk.cpu().numpy(), "dv": dv.cpu().numpy(),
                    "dalpha": dal.cpu().numpy()}


def _check(q, k, v, kept, alpha, do, bq, phi):
    status, got = _run(q, k, v, kept, alpha, do, bq, phi)
    assert status == 0
    kind = "softmax" if phi == sla.SLA_PHI_SOFTMAX else "elu1"
    f64 = lambda t: t.to(torch.float64).numpy()
    ref = orc.sla2_backward(f64(q), f64(k), f64(v), kept, f64(alpha), f64(do), bq, 64, kind)
    for name in ("dq", "dk", "dv", "dalpha"):
        _close(name, got[name], ref[name], _tensor_core(q, bq))


def test_backward_tiny_workload():
    """The small SLA2 case (fp32, d = 64, b_q = 64, 4 of 16 blocks kept)."""
    w = inputs.WORKLOADS["tiny"]
    x = inputs.make_inputs(w)
    g = torch.Generator().manual_seed(5)
    do = torch.randn(x["q"].shape, generator=g).to(x["q"].dtype)
    kept = _kept(5, w.B, w.H, w.n_q, w.n_kv, 4)
    _check(x["q"], x["k"], x["v"], kept, x["alpha"], do, w.bq, sla.SLA_PHI_ELU1)


@pytest.mark.parametrize("N,d,bq,kk", [(1000, 128, 128, 3), (777, 64, 64, 2), (130, 32, 128, 1), (300, 128, 128, 5),
                                      (129, 128, 128, 1), (1000, 128, 64, 3)])
def test_backward_bf16_ragged(N, d, bq, kk):
    """bf16 inputs, ragged last query and key blocks; d = 128 with b_q = 128
    takes the tensor-core kernels (k = n_kv and one ragged row among them)."""
    q, k, v, do, alpha, kept = _case(N + kk, 1, 2, N, d, bq, kk, torch.bfloat16)
    _check(q, k, v, kept, alpha, do, bq, sla.SLA_PHI_ELU1)


@pytest.mark.parametrize("d,bq", [(64, 64), (128, 128)])
def test_backward_softmax_feature_map(d, bq):
    q, k, v, do, alpha, kept = _case(31, 1, 2, 700, d, bq, 3, torch.bfloat16)
    _check(q, k, v, kept, alpha, do, bq, sla.SLA_PHI_SOFTMAX)


def test_backward_tensor_core_is_deterministic_and_matches_the_fp32_kernels():
    """The tensor-core path writes every gradient once in a fixed order: two
    runs agree bit for bit.  The same values as fp32 inputs take the CUDA-core
    path; the two agree within the tensor-core bound."""
    q, k, v, do, alpha, kept = _case(77, 2, 3, 1500, 128, 128, 4, torch.bfloat16)
    s1, a1 = _run(q, k, v, kept, alpha, do, 128, sla.SLA_PHI_ELU1)
    s2, a2 = _run(q, k, v, kept, alpha, do, 128, sla.SLA_PHI_ELU1)
    assert s1 == 0 and s2 == 0
    for name in a1:
        assert np.array_equal(a1[name], a2[name]), name
    s3, f = _run(q.float(), k.float(), v.float(), kept, alpha, do.float(), 128, sla.SLA_PHI_ELU1)
    assert s3 == 0
    for name in a1:
        _close(name, a1[name], f[name], True)


@pytest.mark.parametrize("kk,d,bq", [(0, 32, 64), (5, 32, 64), (0, 128, 128), (5, 128, 128)])
def test_backward_no_block_and_every_block(kk, d, bq):
    """k = 0 (linear branch only) and k = n_kv (sparse branch only, O_l = 0), on
    both paths (d = 128 with b_q = 128 is the tensor-core one)."""
    q, k, v, do, alpha, kept = _case(40 + kk, 2, 1, 300, d, bq, kk, torch.bfloat16)
    _check(q, k, v, kept, alpha, do, bq, sla.SLA_PHI_ELU1)


def test_backward_tensor_core_short_sequence():
    """N below one query tile and one key block short of a second: a single
    ragged tile on both sides."""
    q, k, v, do, alpha, kept = _case(88, 1, 3, 100, 128, 128, 1, torch.bfloat16)
    _check(q, k, v, kept, alpha, do, 128, sla.SLA_PHI_ELU1)
    _check(q, k, v, kept, alpha, do, 128, sla.SLA_PHI_SOFTMAX)


def test_backward_reports_out_of_range_block():
    q, k, v, do, alpha, kept = _case(50, 1, 1, 256, 64, 64, 2, torch.bfloat16)
    kept[0, 0, 1, 1] = 4  # n_kv = 4
    status, got = _run(q, k, v, kept, alpha, do, 64, sla.SLA_PHI_ELU1)
    assert status == 7  # SLA_ERR_DEVICE_INDEX; the block is skipped
    assert all(np.isfinite(t).all() for t in got.values())


def test_backward_wan13_sampled_query_blocks():
    """The full 1.3B-shape backward (12 heads, N = 32760, d = 128, 15 of 512
    key blocks kept by the router): dQ and dalpha of sampled query blocks
    against the oracle.  A query block's dQ rows and its dalpha depend on that
    block alone, so the oracle computes just those blocks (its blocks= path);
    the bound is relative to the largest entry of the checked rows."""
    w = inputs.WORKLOADS["wan13"]
    x = inputs.make_inputs(w)
    kk = w.keep_count if w.keep_count is not None else orc.keep_count(w.keep_ratio, w.n_kv)
    kept, _, _ = orc.route(x["q"].float().numpy(), x["k"].float().numpy(), x["wq"].numpy(), x["wk"].numpy(),
                           w.bq, w.bkv, "sla2", kk)
    g = torch.Generator().manual_seed(13)
    do = torch.randn(x["q"].shape, generator=g).to(torch.bfloat16)
    status, got = _run(x["q"], x["k"], x["v"], kept, x["alpha"], do, w.bq, sla.SLA_PHI_ELU1)
    assert status == 0
    rng = np.random.default_rng(13)
    blocks = [(0, h, int(i)) for h in (0, 6, 11) for i in sorted({0, w.n_q - 1, *rng.integers(0, w.n_q, 2)})]
    f64 = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    ref = orc.sla2_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), kept, f64(x["alpha"]), f64(do), w.bq, w.bkv,
                            blocks=blocks)
    sel = [(b, h, slice(i * w.bq, min((i + 1) * w.bq, w.N))) for (b, h, i) in blocks]
    g_q = np.concatenate([got["dq"][b, h, r] for (b, h, r) in sel])
    r_q = np.concatenate([ref["dq"][b, h, r] for (b, h, r) in sel])
    _close("dq", g_q, r_q, True)
    ga = np.array([got["dalpha"][b, h, i] for (b, h, i) in blocks])
    ra = np.array([ref["dalpha"][b, h, i] for (b, h, i) in blocks])
    _close("dalpha", ga, ra, True)


# ---------------------------------------------------------------- SLA (three labels, W_proj)

def _labels(seed, B, H, nq, nkv, kh, kl):
    """Per query block: kh critical and kl negligible blocks drawn at random."""
    g = np.random.default_rng(seed)
    lab = np.zeros((B, H, nq, nkv), dtype=np.int8)
    for idx in np.ndindex(B, H, nq):
        perm = g.permutation(nkv)
        lab[idx][perm[:kh]] = 1
        lab[idx][perm[kh:kh + kl]] = -1
    return lab


def _run_sla(q, k, v, labels, wp, do, bq, phi):
    dev = "cuda"
    qd, kd, vd, dod = (t.to(dev).contiguous() for t in (q, k, v, do))
    shape = sla.make_shape(qd, bq, 64)
    B, H, N, d = q.shape
    ws = torch.zeros(sla.sla_attn_bwd_workspace_size(shape), dtype=torch.uint8, device=dev)
    dq = torch.full((B, H, N, d), float("nan"), device=dev)
    dk = torch.full_like(dq, float("nan"))
    dv = torch.full_like(dq, float("nan"))
    dwp = torch.full((d, d), float("nan"), device=dev)
    sla.sla_attn_bwd(shape, qd, kd, vd, torch.from_numpy(labels).to(dev).contiguous(), wp.to(dev).contiguous(), phi,
                     dod, dq, dk, dv, dwp, ws)
    status = sla.sla_read_device_status(ws)
    return status, {"dq": dq.cpu().numpy(), "dk": dk.cpu().numpy(), "dv": dv.cpu().numpy(),
                    "dwproj": dwp.cpu().numpy()}


def _check_sla(q, k, v, labels, wp, do, bq, phi, blocks=None):
    status, got = _run_sla(q, k, v, labels, wp, do, bq, phi)
    assert status == 0
    kind = "softmax" if phi == sla.SLA_PHI_SOFTMAX else "elu1"
    f64 = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    ref = orc.sla_backward(f64(q), f64(k), f64(v), labels, f64(wp), f64(do), bq, 64, kind, blocks=blocks)
    for name in ("dq", "dk", "dv", "dwproj"):
        g, r = got[name], ref[name]
        assert np.isfinite(g).all(), name
        scale = max(np.abs(r).max(), 1e-30)
        err = np.abs(g - r).max() / scale
        assert err <= TOL_BWD_REL, (name, err)
    return got


def _wproj(seed, d):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(d, d, generator=g) / d ** 0.5).to(torch.bfloat16)


def test_sla_backward_tiny_workload():
    """The small case (fp32, d = 64, b_q = 64) with the oracle router's SLA
    labels: 2 critical and 3 negligible of 16 blocks per query block."""
    w = inputs.WORKLOADS["tiny"]
    x = inputs.make_inputs(w)
    _, labels, _ = orc.route(x["q"].numpy(), x["k"].numpy(), x["wq"].numpy(), x["wk"].numpy(), w.bq, w.bkv, "sla",
                             2, 3)
    g = torch.Generator().manual_seed(6)
    do = torch.randn(x["q"].shape, generator=g).to(x["q"].dtype)
    _check_sla(x["q"], x["k"], x["v"], labels, x["wproj"], do, w.bq, sla.SLA_PHI_ELU1)


@pytest.mark.parametrize("N,d,bq,kh,kl,phi", [(1000, 128, 128, 3, 4, 0), (777, 64, 64, 2, 3, 0),
                                              (130, 32, 128, 1, 1, 0), (700, 64, 64, 3, 2, 1)])
def test_sla_backward_bf16_ragged(N, d, bq, kh, kl, phi):
    """bf16 inputs, ragged last query and key blocks, both feature maps."""
    q, k, v, do, _, _ = _case(N + kh + 7 * kl, 1, 2, N, d, bq, 0, torch.bfloat16)
    labels = _labels(N + kh, 1, 2, -(-N // bq), -(-N // 64), kh, kl)
    _check_sla(q, k, v, labels, _wproj(N, d), do, bq, phi)


@pytest.mark.parametrize("kh,kl", [(5, 0), (0, 0), (0, 5), (0, 2), (4, 1)])
def test_sla_backward_degenerate_labels(kh, kl):
    """Every block critical (O_l = 0, dW_proj = 0), every block marginal
    (linear only), every block negligible (O = 0, all gradients 0), no critical
    block, no marginal block."""
    q, k, v, do, _, _ = _case(60 + kh + kl, 2, 1, 300, 32, 64, 0, torch.bfloat16)
    labels = _labels(kh * 7 + kl, 2, 1, 5, 5, kh, kl)
    got = _check_sla(q, k, v, labels, _wproj(3, 32), do, 64, sla.SLA_PHI_ELU1)
    if kh + kl == 5:
        assert not got["dwproj"].any()
    if kh == 0 and kl == 5:
        assert not any(t.any() for t in got.values())


def test_sla_backward_reports_bad_label():
    q, k, v, do, _, _ = _case(70, 1, 1, 256, 64, 64, 0, torch.bfloat16)
    labels = _labels(70, 1, 1, 4, 4, 1, 1)
    labels[0, 0, 2, 3] = 2
    status, got = _run_sla(q, k, v, labels, _wproj(4, 64), do, 64, sla.SLA_PHI_ELU1)
    assert status == 7  # SLA_ERR_DEVICE_INDEX; the block counts as marginal
    assert all(np.isfinite(t).all() for t in got.values())


def _sampled_blocks(w, heads, seed):
    rng = np.random.default_rng(seed)
    return [(0, h, int(i)) for h in heads for i in sorted({0, w.n_q - 1, *rng.integers(0, w.n_q, 2)})]


def _do_on_blocks(w, blocks, seed):
    """An upstream gradient that is zero outside the given query blocks, so
    that every key-side gradient and dW_proj are those blocks' shares alone."""
    g = torch.Generator().manual_seed(seed)
    do = torch.zeros(w.B, w.H, w.N, w.d, dtype=torch.bfloat16)
    for (b, h, i) in blocks:
        r = slice(i * w.bq, min((i + 1) * w.bq, w.N))
        do[b, h, r] = torch.randn(do[b, h, r].shape, generator=g).to(torch.bfloat16)
    return do


def test_sla_backward_sla13_full_gradients_of_sampled_blocks():
    """The 1.3B-shape SLA backward (12 heads, N = 32760, d = 128, 26 critical and
    51 negligible of 512 key blocks from the oracle router) with dO non-zero
    on sampled query blocks only, the first and the ragged last among them:
    then dQ, dK, dV and dW_proj over the whole tensors are those blocks'
    shares, which the oracle's blocks= path computes in full."""
    w = inputs.WORKLOADS["sla13"]
    x = inputs.make_inputs(w)
    kh, kl = orc.keep_count(w.crit_ratio, w.n_kv), orc.keep_count(w.negl_ratio, w.n_kv)
    _, labels, _ = orc.route(x["q"].float().numpy(), x["k"].float().numpy(), x["wq"].numpy(), x["wk"].numpy(),
                             w.bq, w.bkv, "sla", kh, kl)
    blocks = _sampled_blocks(w, (0, 11), 21)
    do = _do_on_blocks(w, blocks, 21)
    _check_sla(x["q"], x["k"], x["v"], labels, x["wproj"], do, w.bq, sla.SLA_PHI_ELU1, blocks=blocks)


def test_backward_wan13_full_key_gradients_of_sampled_blocks():
    """The SLA2 counterpart at the 1.3B shape: dO non-zero on sampled query
    blocks only, so dK, dV (whole tensors), dQ and dalpha are the oracle's
    blocks= result in full."""
    w = inputs.WORKLOADS["wan13"]
    x = inputs.make_inputs(w)
    kk = orc.keep_count(w.keep_ratio, w.n_kv)
    kept, _, _ = orc.route(x["q"].float().numpy(), x["k"].float().numpy(), x["wq"].numpy(), x["wk"].numpy(),
                           w.bq, w.bkv, "sla2", kk)
    blocks = _sampled_blocks(w, (3, 9), 22)
    do = _do_on_blocks(w, blocks, 22)
    status, got = _run(x["q"], x["k"], x["v"], kept, x["alpha"], do, w.bq, sla.SLA_PHI_ELU1)
    assert status == 0
    f64 = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    ref = orc.sla2_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), kept, f64(x["alpha"]), f64(do), w.bq, w.bkv,
                            blocks=blocks)
    for name in ("dq", "dk", "dv", "dalpha"):
        _close(name, got[name], ref[name], True)
