"""SoftTop-k router mask (sla_route_soft) on a B200 against the CPU oracle.

"SLA2 深度解读 …" (jefxiong.cn) §06, Stage 1: M_ij = sigmoid(P_c_ij / tau + lambda_i),
tau = 0.1, lambda_i by bisection so that each row's soft selections sum to the
budget.  The scores themselves are bit-exact with the oracle (the router tests).

Tolerance, from the fp32 arithmetic of the kernel: a sigmoid carries a few ulp
of relative error, and a lane-ordered fp32 row sum of n of them (values <= 1,
total k) is off by at most about (n / 32 + 5) * 2^-24 * k, i.e. ~1e-4 for
n <= 1182 and k <= 35.  The kernel's lambda is the exact root for a row sum off
by that much; because sum_j dM_j = df and every dM_j has the same sign, each
entry moves by at most |df|.  The tests allow 5e-4 per entry and 1e-3 on each
row sum, and require the kernel's lambda to solve the oracle's fp64 equation
to within 1e-3.
"""
import numpy as np
import pytest
import torch

from oracle import sla_oracle as orc
from sparse_linear_attention_b200 import inputs, sla
from tests.gpu_common import as32, run_route_soft

pytestmark = pytest.mark.gpu

TOL_M = 5e-4
TOL_SUM = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    sla.lib()


def _check(q, k, wq, wk, bq, bkv, kk, tau):
    mask, lam = run_route_soft(q, k, wq, wk, bq, bkv, kk, tau)
    _, _, s = orc.route(as32(q), as32(k), None if wq is None else wq.numpy(), None if wk is None else wk.numpy(),
                        bq, bkv, "sla2", 0)
    om, _ = orc.soft_topk(s, kk, tau=tau)
    n = s.shape[-1]
    assert np.isfinite(mask).all()
    err = np.abs(mask - om).max()
    assert err <= TOL_M, f"max |M - M_oracle| = {err:.3e}"
    serr = np.abs(mask.sum(-1, dtype=np.float64) - kk).max()
    assert serr <= TOL_SUM, f"max |row sum - k| = {serr:.3e}"
    if 0 < kk < n:
        f = orc.sigmoid(s.astype(np.float64) / tau + lam.astype(np.float64)[..., None]).sum(-1)
        ferr = np.abs(f - kk).max()
        assert ferr <= TOL_SUM, f"lambda misses the budget by {ferr:.3e}"
    elif kk == 0:
        assert (mask == 0).all() and np.isneginf(lam).all()
    else:
        assert (mask == 1).all() and np.isposinf(lam).all()
    return err


@pytest.mark.parametrize("name", ["tiny", "wan13"])
def test_soft_topk_workloads(name):
    w = inputs.WORKLOADS[name]
    x = inputs.make_inputs(w)
    kk = w.keep_count if w.keep_count is not None else orc.keep_count(w.keep_ratio, w.n_kv)
    _check(x["q"], x["k"], x["wq"], x["wk"], w.bq, w.bkv, kk, 0.1)


def test_soft_topk_many_key_blocks():
    """n_kv > 1024: the largest per-lane register layout; identity projections."""
    g = torch.Generator().manual_seed(11)
    q = torch.randn(1, 1, 70000, 64, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 1, 70000, 64, generator=g).to(torch.bfloat16)
    _check(q, k, None, None, 128, 64, 33, 0.1)


@pytest.mark.parametrize("kk,tau", [(0, 0.1), (16, 0.1), (1, 0.05), (5, 1.0), (15, 0.02)])
def test_soft_topk_budgets_and_temperatures(kk, tau):
    """Ragged N, d = 40, the empty and the full budget, several temperatures."""
    g = torch.Generator().manual_seed(100 + kk)
    N, d = 1000, 40
    q = (torch.randn(1, 2, N, d, generator=g) * 1.5).to(torch.bfloat16)
    k = (torch.randn(1, 2, N, d, generator=g) * 1.5).to(torch.bfloat16)
    wq = torch.randn(d, d, generator=g) / d ** 0.5
    wk = torch.randn(d, d, generator=g) / d ** 0.5
    _check(q, k, wq, wk, 128, 64, kk, tau)
