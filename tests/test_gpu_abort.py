"""Device-side failure detection of the attention kernel on a B200.

Every wait in the kernel is bounded.  The test hook SLA_FLAG_WAIT_TEST sets
the limit to zero, so the first wait that is not already satisfied gives up,
as a wait that ran out would; nothing is left unsatisfied on purpose.  The
kernel must then stop, drain the copies and products it started, free its
tensor memory and return: the call reports SLA_ERR_TIMEOUT through the
status word, and the same process can run the forward again with the exact
result of a clean run.  The check runs in a child process so that the test
session survives whatever happens there.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CHILD = r'''
import sys
sys.path.insert(0, {root!r})
import numpy as np
import torch
from sparse_linear_attention_b200 import inputs, sla
w = inputs.Workload("abort", 1, 2, (1, 1, 2000), 128, 128, 64, "bf16", keep_count=3)
x = inputs.random_inputs(1, 2, 2000, 128, dtype="bf16", seed=17, scale=1.5, n_q=w.n_q)
dev = "cuda"
q, k, v = x["q"].to(dev), x["k"].to(dev), x["v"].to(dev)
shape = sla.make_shape(q, w.bq, w.bkv)
ws = torch.zeros(sla.sla_workspace_size(shape, {mode}), dtype=torch.uint8, device=dev)
kept = torch.empty(1, 2, w.n_q, 3, dtype=torch.int32, device=dev)
sla.sla_route(shape, q, k, x["wq"].to(dev), x["wk"].to(dev), 0, 3, 0, kept, None, None, ws)
alpha = x["alpha"].to(dev)
def forward(flags):
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device=dev)
    sla.sla2_attn_fwd(shape, q, k, v, kept, 3, alpha, 0, flags, out, ws)
    return sla.sla_read_device_status(ws), out.cpu().numpy()
st0, ref = forward({low})
assert st0 == 0, st0
st1, _ = forward({low} | sla.SLA_FLAG_WAIT_TEST)
assert st1 == 6, ("expected SLA_ERR_TIMEOUT", st1)
st2, again = forward({low})
assert st2 == 0, st2
assert np.array_equal(ref.view(np.uint32), again.view(np.uint32))
print("ABORT_PATH_OK")
'''


@pytest.mark.parametrize("low", ["0", "sla.SLA_FLAG_FP8"])
def test_wait_limit_zero_reports_timeout_and_leaves_the_device_usable(low):
    mode = "sla.SLA_WS_FP8" if low != "0" else "0"
    code = _CHILD.format(root=ROOT, mode=mode, low=low)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and "ABORT_PATH_OK" in out.stdout, (out.stdout[-1500:], out.stderr[-3000:])
