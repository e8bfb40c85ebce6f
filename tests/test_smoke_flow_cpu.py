"""__graft_entry__.smoke()'s call sequence on the CPU, with the library's
binding replaced by stand-ins that fill every output from the oracle.  This
checks the smoke's own flow (calls, argument order, shapes, the comparisons);
the kernels themselves are checked by the -m gpu tests."""
import sys
import types

import torch

import __graft_entry__ as ge
import sparse_linear_attention_b200 as pkg
from oracle import sla_oracle as orc
from sparse_linear_attention_b200 import sla as real


def _fake_binding(calls):
    fake = types.ModuleType("sla")
    for n in dir(real):
        if n.startswith("SLA_") or n in ("STATUS_NAMES", "make_shape", "Shape"):
            setattr(fake, n, getattr(real, n))

    def route(shape, q, k, wq, wk, mode, kk, kn, kept, labels, scores, ws, stream=None):
        calls.append("route")
        o, _, _ = orc.route(q.float().numpy(), k.float().numpy(), wq.numpy(), wk.numpy(), shape.bq, shape.bkv,
                            "sla2", kk)
        kept.copy_(torch.from_numpy(o))

    def fwd(shape, q, k, v, kept, kk, alpha, phi, flags, out, ws, stream=None):
        calls.append("fwd")
        o = orc.sla2_forward(q.double().numpy(), k.double().numpy(), v.double().numpy(), kept.numpy(),
                             alpha.numpy(), shape.bq, shape.bkv)["o"]
        out.copy_(torch.from_numpy(o))

    def bwd(shape, q, k, v, kept, kk, alpha, phi, dout, dq, dk, dv, dal, ws, stream=None):
        calls.append("bwd")
        assert dout.shape == q.shape == dq.shape == dk.shape == dv.shape and dal.shape == alpha.shape
        assert dout.dtype == q.dtype and kk == kept.shape[-1]
        g = orc.sla2_backward(q.double().numpy(), k.double().numpy(), v.double().numpy(), kept.numpy(),
                              alpha.double().numpy(), dout.double().numpy(), shape.bq, shape.bkv)
        for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv"), (dal, "dalpha")):
            t.copy_(torch.from_numpy(g[n]))

    fake.sla_workspace_size = lambda shape, mode=0: 256
    fake.sla2_attn_bwd_workspace_size = lambda shape: 256
    fake.sla_route, fake.sla2_attn_fwd, fake.sla2_attn_bwd = route, fwd, bwd
    fake.sla_prepare = lambda *a, **kw: calls.append("prepare")
    fake.sla_read_device_status = lambda ws, stream=None: 0
    return fake


def test_smoke_flow(monkeypatch, capsys):
    calls = []
    fake = _fake_binding(calls)
    monkeypatch.setattr(pkg, "sla", fake)
    monkeypatch.setitem(sys.modules, "sparse_linear_attention_b200.sla", fake)
    cpu = torch.device("cpu")
    monkeypatch.setattr(torch, "device", lambda *a, **kw: cpu)
    ge.smoke()
    assert calls == ["route", "fwd", "bwd", "prepare", "route", "fwd"]
    assert "smoke ok" in capsys.readouterr().out
