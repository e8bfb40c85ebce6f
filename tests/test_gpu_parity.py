"""libsla on a B200 against the CPU oracle, on the same seeded inputs.

Masks and scores must match bit for bit; outputs within max-abs 2e-3 and
relative L1 1e-2 of the fp64 oracle (bf16 tensor-core arithmetic)."""
import numpy as np
import pytest
import torch

from oracle import sla_oracle as orc
from sparse_linear_attention_b200 import inputs, sla
from tests.gpu_common import (TOL_BF16, as32, as64, compare, run_route, run_route_after_prepare, run_sla, run_sla2,
                              sample_blocks)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    sla.lib()


_CACHE = {}


def workload(name):
    if name not in _CACHE:
        w = inputs.WORKLOADS[name]
        _CACHE[name] = (w, inputs.make_inputs(w))
    return _CACHE[name]


def k_of(w):
    return w.keep_count if w.keep_count is not None else orc.keep_count(w.keep_ratio, w.n_kv)


# ------------------------------------------------------------------ router

@pytest.mark.parametrize("name", ["tiny", "wan13", "wan14"])
@pytest.mark.parametrize("proj", [True, False])
def test_route_sla2_bitexact(name, proj):
    w, x = workload(name)
    kk = k_of(w)
    wq, wk = (x["wq"], x["wk"]) if proj else (None, None)
    kept, lab, sc = run_route(x["q"], x["k"], wq, wk, w.bq, w.bkv, sla.SLA_MODE_SLA2_TOPK, kk)
    okept, olab, osc = orc.route(as32(x["q"]), as32(x["k"]), None if wq is None else wq.numpy(),
                                 None if wk is None else wk.numpy(), w.bq, w.bkv, "sla2", kk)
    assert np.array_equal(sc.view(np.uint32), osc.view(np.uint32)), "scores differ"
    assert np.array_equal(kept, okept), f"{int((kept != okept).sum())} kept indices differ"
    assert np.array_equal(lab, olab)


def test_route_sla_three_way_bitexact():
    w, x = workload("sla13")
    kh, kl = orc.keep_count(w.crit_ratio, w.n_kv), orc.keep_count(w.negl_ratio, w.n_kv)
    kept, lab, sc = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, sla.SLA_MODE_SLA_3WAY, kh, kl)
    okept, olab, osc = orc.route(as32(x["q"]), as32(x["k"]), x["wq"].numpy(), x["wk"].numpy(), w.bq, w.bkv,
                                 "sla", kh, kl)
    assert np.array_equal(sc.view(np.uint32), osc.view(np.uint32))
    assert np.array_equal(kept, okept)
    assert np.array_equal(lab, olab)
    assert ((lab == 1).sum(-1) == kh).all() and ((lab == -1).sum(-1) == kl).all()


@pytest.mark.parametrize("N,d,mode", [(1000, 40, 0), (777, 24, 1), (300, 128, 1)])
def test_route_bitexact_odd_shapes(N, d, mode):
    """Head dims that are not a multiple of 16 (the score kernel feeds 16-channel
    slices), n_kv not a multiple of 4 (padded key rows), ragged tails, both modes."""
    g = torch.Generator().manual_seed(N + d)
    B, H = 1, 3
    q = (torch.randn(B, H, N, d, generator=g) * 1.5).to(torch.bfloat16)
    k = (torch.randn(B, H, N, d, generator=g) * 1.5).to(torch.bfloat16)
    wq = torch.randn(d, d, generator=g) / d ** 0.5
    wk = torch.randn(d, d, generator=g) / d ** 0.5
    nkv = -(-N // 64)
    kh, kl = min(3, nkv), (min(2, nkv - 3) if mode == 1 else 0)
    kept, lab, sc = run_route(q, k, wq, wk, 128, 64, mode, kh, kl)
    okept, olab, osc = orc.route(as32(q), as32(k), wq.numpy(), wk.numpy(), 128, 64, "sla" if mode else "sla2", kh, kl)
    assert np.array_equal(sc.view(np.uint32), osc.view(np.uint32)), "scores differ"
    assert np.array_equal(kept, okept)
    assert np.array_equal(lab, olab)


@pytest.mark.parametrize("name,mode", [("wan13", 0), ("sla13", 1)])
def test_route_key_means_from_prepare_bitexact(name, mode):
    """The router with the key-block means the prepass wrote (K read once):
    the same bits as the oracle's own pooling."""
    w, x = workload(name)
    if mode == 0:
        kh, kl = k_of(w), 0
    else:
        kh, kl = orc.keep_count(w.crit_ratio, w.n_kv), orc.keep_count(w.negl_ratio, w.n_kv)
    kept, lab, sc = run_route_after_prepare(x["q"], x["k"], x["v"], x["wq"], x["wk"], w.bq, w.bkv, mode, kh, kl)
    okept, olab, osc = orc.route(as32(x["q"]), as32(x["k"]), x["wq"].numpy(), x["wk"].numpy(), w.bq, w.bkv,
                                 "sla" if mode else "sla2", kh, kl)
    assert np.array_equal(sc.view(np.uint32), osc.view(np.uint32)), "scores differ"
    assert np.array_equal(kept, okept)
    assert np.array_equal(lab, olab)


def test_route_key_means_from_prepare_ragged():
    """A ragged last key block (N = 1000: 40 tokens) and no projections."""
    g = torch.Generator().manual_seed(5)
    q, k, v = ((torch.randn(1, 2, 1000, 128, generator=g) * 1.5).to(torch.bfloat16) for _ in range(3))
    kept, lab, sc = run_route_after_prepare(q, k, v, None, None, 128, 64, 0, 4)
    okept, olab, osc = orc.route(as32(q), as32(k), None, None, 128, 64, "sla2", 4)
    assert np.array_equal(sc.view(np.uint32), osc.view(np.uint32))
    assert np.array_equal(kept, okept)


def test_route_key_means_from_prepare_needs_bf16_d128():
    q = torch.zeros(1, 1, 256, 64, dtype=torch.bfloat16)
    with pytest.raises(sla.SLAError) as e:
        run_route_after_prepare(q, q, q, None, None, 64, 64, 0, 2)
    assert e.value.status == 2  # SLA_ERR_UNSUPPORTED


def test_route_ties_break_to_lower_index():
    # identical key blocks -> equal scores; the lower block index must win
    B, H, N, d = 1, 1, 512, 64
    q = torch.randn(B, H, N, d).to(torch.bfloat16)
    k = torch.randn(B, H, 64, d).repeat(1, 1, N // 64, 1).to(torch.bfloat16)
    kept, _, sc = run_route(q, k, None, None, 64, 64, 0, 3)
    assert np.all(kept == np.arange(3))
    assert np.all(sc == sc[..., :1])


# ------------------------------------------------------------------ SLA2 attention

def _sla2_check(w, x, kept, blocks=None, phi=sla.SLA_PHI_ELU1, out_dtype=torch.float32, tol=TOL_BF16):
    got = run_sla2(x["q"], x["k"], x["v"], kept, x["alpha"], w.bq, w.bkv, phi, out_dtype)
    kind = "elu1" if phi == sla.SLA_PHI_ELU1 else "softmax"
    want = orc.sla2_forward(as64(x["q"]), as64(x["k"]), as64(x["v"]), kept, x["alpha"].numpy(), w.bq, w.bkv,
                            kind, blocks=blocks)["o"]
    if blocks is None:
        blocks = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(w.n_q)]
    return compare(got, want, blocks, w.bq, tol=tol)


def test_sla2_tiny_all_rows():
    w, x = workload("tiny")
    kept, _, _ = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, 0, k_of(w))
    _sla2_check(w, x, kept)


def test_sla2_wan13_sampled_blocks():
    w, x = workload("wan13")
    kept, _, _ = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, 0, k_of(w))
    _sla2_check(w, x, kept, blocks=sample_blocks(w.B, w.H, w.n_q, 4))


def test_sla2_wan14_sampled_blocks():
    """Full 14B-shape launch; the oracle checks 4 heads x 4 query blocks."""
    w, x = workload("wan14")
    kk = k_of(w)
    kept, _, _ = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, 0, kk)
    got = run_sla2(x["q"], x["k"], x["v"], kept, x["alpha"], w.bq, w.bkv)
    hs = [0, 13, 26, 39]
    sub = lambda t: t[:, hs]  # noqa: E731
    blocks = sample_blocks(1, len(hs), w.n_q, 4, seed=1)
    want = orc.sla2_forward(as64(sub(x["q"])), as64(sub(x["k"])), as64(sub(x["v"])), kept[:, hs],
                            x["alpha"][:, hs].numpy(), w.bq, w.bkv, blocks=blocks)["o"]
    compare(got[:, hs], want, blocks, w.bq)


def _rand_case(N, d, dtype="bf16", B=1, H=2, bq=128, seed=3, scale=1.0):
    w = inputs.Workload("case", B, H, (1, 1, N), d, bq, 64, dtype, keep_count=1)
    x = inputs.random_inputs(B, H, N, d, dtype=dtype, seed=seed, scale=scale, n_q=w.n_q)
    return w, x


def _rand_kept(w, k, seed=0):
    rng = np.random.default_rng(seed)
    return np.stack([np.sort(rng.choice(w.n_kv, k, replace=False)) for _ in range(w.B * w.H * w.n_q)]
                    ).reshape(w.B, w.H, w.n_q, k).astype(np.int32)


@pytest.mark.parametrize("N,d,bq", [(200, 128, 128), (1000, 64, 64), (777, 128, 64), (64, 128, 128),
                                    (1, 128, 128), (4100, 96, 128)])
def test_sla2_ragged_shapes(N, d, bq):
    w, x = _rand_case(N, d, bq=bq, scale=1.5)
    kk = max(1, min(3, w.n_kv - 1)) if w.n_kv > 1 else 1
    _sla2_check(w, x, _rand_kept(w, kk))


def test_sla2_no_block_kept_is_linear_attention():
    w, x = _rand_case(1000, 128)
    _sla2_check(w, x, np.zeros((1, 2, w.n_q, 0), np.int32))


def test_sla2_every_block_kept():
    w, x = _rand_case(1000, 128, scale=1.5)
    kept = np.broadcast_to(np.arange(w.n_kv, dtype=np.int32), (1, 2, w.n_q, w.n_kv))
    _sla2_check(w, x, kept)


def test_sla2_softmax_feature_map():
    w, x = workload("tiny")
    kept, _, _ = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, 0, k_of(w))
    _sla2_check(w, x, kept, phi=sla.SLA_PHI_SOFTMAX)


def test_sla2_softmax_feature_map_production_path():
    """Softmax-phi on the bf16 d = 128 path the benchmark times: the TMA
    prepass (phi = softmax), the router on the prepass's key-block means, the
    attention kernel on the prepared totals; sampled query blocks of the
    full-size 1.3B-shape launch."""
    w, x = workload("wan13")
    kk = k_of(w)
    dev = "cuda"
    qd, kd, vd = x["q"].to(dev), x["k"].to(dev), x["v"].to(dev)
    shape = sla.make_shape(qd, w.bq, w.bkv)
    ws = torch.zeros(sla.sla_workspace_size(shape, 0), dtype=torch.uint8, device=dev)
    kept = torch.full((w.B, w.H, w.n_q, kk), -7, dtype=torch.int32, device=dev)
    out = torch.full(x["q"].shape, float("nan"), dtype=torch.float32, device=dev)
    sla.sla_prepare(shape, kd, vd, sla.SLA_PHI_SOFTMAX, ws)
    sla.sla_route(shape, qd, kd, x["wq"].to(dev), x["wk"].to(dev),
                  sla.SLA_MODE_SLA2_TOPK | sla.SLA_ROUTE_KBAR_FROM_WS, kk, 0, kept, None, None, ws)
    sla.sla2_attn_fwd(shape, qd, kd, vd, kept, kk, x["alpha"].to(dev), sla.SLA_PHI_SOFTMAX, sla.SLA_FLAG_PREPARED,
                      out, ws)
    assert sla.sla_read_device_status(ws) == 0
    kept_h = kept.cpu().numpy()
    okept, _, _ = orc.route(as32(x["q"]), as32(x["k"]), x["wq"].numpy(), x["wk"].numpy(), w.bq, w.bkv, "sla2", kk)
    assert np.array_equal(kept_h, okept)
    blocks = sample_blocks(w.B, w.H, w.n_q, 3, seed=6)
    want = orc.sla2_forward(as64(x["q"]), as64(x["k"]), as64(x["v"]), kept_h, x["alpha"].numpy(), w.bq, w.bkv,
                            phi_kind="softmax", blocks=blocks)["o"]
    compare(out.cpu().numpy(), want, blocks, w.bq)


def test_sla2_bf16_output():
    w, x = _rand_case(1500, 128, scale=1.5)
    kept = _rand_kept(w, 4)
    got = run_sla2(x["q"], x["k"], x["v"], kept, x["alpha"], w.bq, w.bkv, out_dtype=torch.bfloat16)
    want = orc.sla2_forward(as64(x["q"]), as64(x["k"]), as64(x["v"]), kept, x["alpha"].numpy(), w.bq, w.bkv)["o"]
    # bf16 output rounding adds up to half an ulp of |O|
    assert np.all(np.abs(got - want) <= TOL_BF16 + np.abs(want) * 2.0 ** -8)


def test_sla2_fp32_inputs_off_the_bf16_grid():
    """f32 inputs are rounded to bf16 for the tensor-core stages; against the
    oracle on the rounded values the usual bound holds."""
    B, H, N, d = 1, 2, 900, 128
    g = torch.Generator().manual_seed(11)
    q, k, v = (torch.randn(B, H, N, d, generator=g) * 1.3 for _ in range(3))
    w = inputs.Workload("f32", B, H, (1, 1, N), d, 128, 64, "f32", keep_count=3)
    alpha = torch.rand(B, H, w.n_q, generator=g)
    kept = _rand_kept(w, 3)
    got = run_sla2(q, k, v, kept, alpha, 128, 64)
    r = lambda t: t.to(torch.bfloat16).to(torch.float64).numpy()  # noqa: E731
    want = orc.sla2_forward(r(q), r(k), v.to(torch.float64).numpy(), kept, alpha.numpy(), 128, 64)["o"]
    compare(got, want, [(0, h, i) for h in range(H) for i in range(w.n_q)], 128)


def test_sla2_prepared_flag_and_determinism():
    w, x = _rand_case(3000, 128, scale=1.5)
    kept = _rand_kept(w, 5)
    dev = "cuda"
    shape = sla.make_shape(x["q"].cuda(), w.bq, w.bkv)
    ws = torch.zeros(sla.sla_workspace_size(shape, 0), dtype=torch.uint8, device=dev)
    a = run_sla2(x["q"], x["k"], x["v"], kept, x["alpha"], w.bq, w.bkv, ws=ws)
    b = run_sla2(x["q"], x["k"], x["v"], kept, x["alpha"], w.bq, w.bkv, ws=ws, flags=sla.SLA_FLAG_PREPARED)
    c = run_sla2(x["q"], x["k"], x["v"], kept, x["alpha"], w.bq, w.bkv)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert np.array_equal(a.view(np.uint32), c.view(np.uint32))


# ------------------------------------------------------------------ SLA attention

def _sla_check(w, x, labels, blocks=None):
    got = run_sla(x["q"], x["k"], x["v"], labels, x["wproj"], w.bq, w.bkv)
    want = orc.sla_forward(as64(x["q"]), as64(x["k"]), as64(x["v"]), labels, as64(x["wproj"]), w.bq, w.bkv,
                           blocks=blocks)["o"]
    if blocks is None:
        blocks = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(w.n_q)]
    return compare(got, want, blocks, w.bq)


def test_sla_tiny_all_rows():
    w, x = workload("tiny")
    _, lab, _ = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, 1, 2, 3)
    _sla_check(w, x, lab)


def test_sla_wan13_sampled_blocks():
    w, x = workload("sla13")
    kh, kl = orc.keep_count(w.crit_ratio, w.n_kv), orc.keep_count(w.negl_ratio, w.n_kv)
    _, lab, _ = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, 1, kh, kl)
    _sla_check(w, x, lab, blocks=sample_blocks(w.B, w.H, w.n_q, 3, seed=2))


def test_sla_64x64_sampled_blocks():
    """SLA at the block sizes of its own page: b_q = b_kv = 64."""
    w, x = workload("sla13_64")
    kh, kl = orc.keep_count(w.crit_ratio, w.n_kv), orc.keep_count(w.negl_ratio, w.n_kv)
    _, lab, _ = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, 1, kh, kl)
    _sla_check(w, x, lab, blocks=sample_blocks(w.B, w.H, w.n_q, 3, seed=3))


def test_sla_label_edge_cases():
    w, x = _rand_case(700, 128, scale=1.5)
    rng = np.random.default_rng(5)
    lab = rng.integers(-1, 2, (1, 2, w.n_q, w.n_kv)).astype(np.int8)
    lab[0, 0, 0, :] = 1          # all critical: no linear term
    lab[0, 0, 1, :] = 0          # all marginal: no softmax term
    lab[0, 1, 0, :] = -1         # all negligible: output 0
    lab[0, 1, 1, :] = 0
    lab[0, 1, 1, 0] = -1         # marginal except one negligible block
    _sla_check(w, x, lab)


# ------------------------------------------------------------------ e4m3 sparse branch

def _fp8_check(w, x, kept, blocks=None, heads=None):
    from tests.gpu_common import TOL_FP8
    got = run_sla2(x["q"], x["k"], x["v"], kept, x["alpha"], w.bq, w.bkv, flags=sla.SLA_FLAG_FP8)
    hs = list(range(w.H)) if heads is None else heads
    sub = lambda t: t[:, hs]  # noqa: E731
    want = orc.sla2_forward_fp8(as64(sub(x["q"])), as64(sub(x["k"])), as64(sub(x["v"])), kept[:, hs],
                                x["alpha"][:, hs].numpy(), w.bq, w.bkv, blocks=blocks)["o"]
    if blocks is None:
        blocks = [(0, h, i) for h in range(len(hs)) for i in range(w.n_q)]
    return compare(got[:, hs], want, blocks, w.bq, tol=TOL_FP8)


def test_fp8_tiny_all_rows():
    w, x = workload("tiny")
    kept, _, _ = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, 0, k_of(w))
    _fp8_check(w, x, kept)


@pytest.mark.parametrize("ratio", [0.03, 0.05, 0.10])
def test_fp8_wan13_keep_sweep(ratio):
    w, x = workload("wan13")
    kk = orc.keep_count(ratio, w.n_kv)
    kept, _, _ = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, 0, kk)
    _fp8_check(w, x, kept, blocks=sample_blocks(1, 3, w.n_q, 3, seed=4), heads=[0, 5, 11])


@pytest.mark.parametrize("ratio", [0.03, 0.05, 0.10])
def test_fp8_wan14_keep_sweep(ratio):
    """The e4m3 branch at the 14B shape for the keep sweep of that workload
    (35 / 59 / 118 of 1182 key blocks): full launch, 3 heads x 3 query blocks
    checked."""
    _, x = workload("wan14")  # same seeded inputs as the e4m3 14B workload
    w = inputs.WORKLOADS["fp8_14"]
    kk = orc.keep_count(ratio, w.n_kv)
    kept, _, _ = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, 0, kk)
    _fp8_check(w, x, kept, blocks=sample_blocks(1, 3, w.n_q, 3, seed=5), heads=[0, 21, 39])


@pytest.mark.parametrize("N,d,bq", [(777, 128, 64), (300, 64, 128)])
def test_fp8_ragged_shapes(N, d, bq):
    """Ragged shapes on plain N(0, 1.5^2) inputs (|V| up to 7, peaked rows).
    The kernel quantises P once per softmax step of two kept blocks; the
    oracle's default quantises it once per kept block.  The pages fix no tile,
    so both are readings of the same step, and the grouping moves only the
    rounding of P.  Here that rounding difference alone (the oracle against
    itself, one block vs two per step) reaches 4e-2, above the 3e-2 gate that
    the seeded workloads meet against the per-block oracle.  So the kernel is
    held to the gate against the oracle with its own grouping, and to the gate
    plus the oracle's own grouping spread against the per-block default."""
    from tests.gpu_common import TOL_FP8
    w, x = _rand_case(N, d, bq=bq, scale=1.5)
    kept = _rand_kept(w, min(3, w.n_kv))
    got = run_sla2(x["q"], x["k"], x["v"], kept, x["alpha"], w.bq, w.bkv, flags=sla.SLA_FLAG_FP8)
    args = (as64(x["q"]), as64(x["k"]), as64(x["v"]), kept, x["alpha"].numpy(), w.bq, w.bkv)
    per_block = orc.sla2_forward_fp8(*args)["o"]
    per_step = orc.sla2_forward_fp8(*args, kv_tile=2)["o"]
    spread = float(np.abs(per_block - per_step).max())
    blocks = [(0, h, i) for h in range(w.H) for i in range(w.n_q)]
    compare(got, per_step, blocks, w.bq, tol=TOL_FP8)
    compare(got, per_block, blocks, w.bq, tol=TOL_FP8 + spread)


# ------------------------------------------------------------------ host-buffer entry point

@pytest.mark.parametrize("name,fp8", [("tiny", False), ("smoke128", False), ("smoke128", True)])
def test_forward_host_matches_the_device_calls(name, fp8):
    """sla2_forward_host (host inputs in, host output out, one C-ABI call) runs
    the same kernels as sla_prepare + sla_route + sla2_attn_fwd on device
    buffers: outputs and kept lists identical bit for bit, and the oracle's
    router agrees."""
    if name == "tiny":
        w, x = workload("tiny")
    else:
        w = inputs.Workload("smoke128", 1, 2, (4, 16, 16), 128, 128, 64, "bf16", keep_count=4, seed=3)
        x = inputs.make_inputs(w)
    kk = k_of(w)
    flags = sla.SLA_FLAG_FP8 if fp8 else 0
    dev = "cuda"
    shape = sla.make_shape(x["q"], w.bq, w.bkv)
    hout = torch.full(x["q"].shape, float("nan"), dtype=torch.float32).pin_memory()
    hkept = torch.full((w.B, w.H, w.n_q, kk), -1, dtype=torch.int32).pin_memory()
    pin = {n: x[n].contiguous().pin_memory() for n in ("q", "k", "v", "wq", "wk", "alpha")}
    dbuf = torch.zeros(sla.sla2_forward_host_device_bytes(shape, kk, sla.SLA_F32, flags), dtype=torch.uint8,
                       device=dev)
    sla.sla2_forward_host(shape, pin["q"], pin["k"], pin["v"], pin["wq"], pin["wk"], pin["alpha"], kk,
                          sla.SLA_PHI_ELU1, flags, hout, hkept, dbuf)
    assert sla.sla_read_device_status(dbuf) == 0
    # the same forward through the device-pointer calls
    qd, kd, vd = x["q"].to(dev), x["k"].to(dev), x["v"].to(dev)
    ws = torch.zeros(sla.sla_workspace_size(shape, sla.SLA_WS_FP8 if fp8 else 0), dtype=torch.uint8, device=dev)
    kept = torch.empty(w.B, w.H, w.n_q, kk, dtype=torch.int32, device=dev)
    out = torch.empty(x["q"].shape, dtype=torch.float32, device=dev)
    kbar = w.dtype == "bf16" and w.d == 128
    if kbar:
        sla.sla_prepare(shape, kd, vd, sla.SLA_PHI_ELU1, ws)
    sla.sla_route(shape, qd, kd, x["wq"].to(dev), x["wk"].to(dev), sla.SLA_ROUTE_KBAR_FROM_WS if kbar else 0, kk,
                  0, kept, None, None, ws)
    if not kbar:
        sla.sla_prepare(shape, kd, vd, sla.SLA_PHI_ELU1, ws)
    sla.sla2_attn_fwd(shape, qd, kd, vd, kept, kk, x["alpha"].to(dev), sla.SLA_PHI_ELU1,
                      sla.SLA_FLAG_PREPARED | flags, out, ws)
    assert sla.sla_read_device_status(ws) == 0
    assert np.array_equal(hkept.numpy(), kept.cpu().numpy())
    assert np.array_equal(hout.numpy().view(np.uint32), out.cpu().numpy().view(np.uint32))
    okept, _, _ = orc.route(as32(x["q"]), as32(x["k"]), x["wq"].numpy(), x["wk"].numpy(), w.bq, w.bkv, "sla2", kk)
    assert np.array_equal(hkept.numpy(), okept)


# ------------------------------------------------------------------ INT8 variant of the low-bit branch

def _int8_check(w, x, kept, blocks=None, heads=None, extra_tol=0.0):
    from tests.gpu_common import TOL_FP8
    got = run_sla2(x["q"], x["k"], x["v"], kept, x["alpha"], w.bq, w.bkv, flags=sla.SLA_FLAG_INT8)
    hs = list(range(w.H)) if heads is None else heads
    sub = lambda t: t[:, hs]  # noqa: E731
    args = (as64(sub(x["q"])), as64(sub(x["k"])), as64(sub(x["v"])), kept[:, hs], x["alpha"][:, hs].numpy(),
            w.bq, w.bkv)
    want = orc.sla2_forward_int8(*args, blocks=blocks)["o"]
    if blocks is None:
        blocks = [(0, h, i) for h in range(len(hs)) for i in range(w.n_q)]
    return compare(got[:, hs], want, blocks, w.bq, tol=TOL_FP8 + extra_tol)


def test_int8_tiny_all_rows():
    """INT8 Q, K' (kind::i8 S), e4m3 P, V on the tiny workload, every row."""
    w, x = workload("tiny")
    kept, _, _ = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, 0, k_of(w))
    _int8_check(w, x, kept)


@pytest.mark.parametrize("ratio", [0.03, 0.10])
def test_int8_wan13_sampled_blocks(ratio):
    w, x = workload("wan13")
    kk = orc.keep_count(ratio, w.n_kv)
    kept, _, _ = run_route(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, 0, kk)
    _int8_check(w, x, kept, blocks=sample_blocks(1, 3, w.n_q, 3, seed=7), heads=[0, 4, 9])


@pytest.mark.parametrize("N,d,bq", [(777, 128, 64), (300, 64, 128)])
def test_int8_ragged_shapes(N, d, bq):
    """As test_fp8_ragged_shapes: held to the gate against the oracle with the
    kernel's two-block softmax step, and to the gate plus the oracle's own
    grouping spread against the per-block default."""
    from tests.gpu_common import TOL_FP8
    w, x = _rand_case(N, d, bq=bq, scale=1.5)
    kept = _rand_kept(w, min(3, w.n_kv))
    got = run_sla2(x["q"], x["k"], x["v"], kept, x["alpha"], w.bq, w.bkv, flags=sla.SLA_FLAG_INT8)
    args = (as64(x["q"]), as64(x["k"]), as64(x["v"]), kept, x["alpha"].numpy(), w.bq, w.bkv)
    per_block = orc.sla2_forward_int8(*args)["o"]
    per_step = orc.sla2_forward_int8(*args, kv_tile=2)["o"]
    spread = float(np.abs(per_block - per_step).max())
    blocks = [(0, h, i) for h in range(w.H) for i in range(w.n_q)]
    compare(got, per_step, blocks, w.bq, tol=TOL_FP8)
    compare(got, per_block, blocks, w.bq, tol=TOL_FP8 + spread)


def test_low_bit_flags_exclude_each_other():
    w, x = _rand_case(300, 64, bq=128)
    with pytest.raises(sla.SLAError, match="exclude"):
        run_sla2(x["q"], x["k"], x["v"], _rand_kept(w, 2), x["alpha"], w.bq, w.bkv,
                 flags=sla.SLA_FLAG_INT8 | sla.SLA_FLAG_FP8)
