"""Shared helpers of the GPU parity tests: run libsla through its C ABI and
the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import sla_oracle as orc
from sparse_linear_attention_b200 import sla

# max-abs error allowed between the bf16 tensor-core path and the fp64 oracle
TOL_BF16 = 2e-3
TOL_REL_L1 = 1e-2
# e4m3 sparse branch against the oracle that emulates the same quantisation
TOL_FP8 = 3e-2


def as32(t):
    return t.to(torch.float32).numpy()


def as64(t):
    return t.to(torch.float64).numpy()


def run_route(q, k, wq, wk, bq, bkv, mode, k_keep, k_neg=0):
    dev = "cuda"
    qd, kd = q.to(dev), k.to(dev)
    shape = sla.make_shape(qd, bq, bkv)
    B, H, N, d = q.shape
    nq, nkv = -(-N // bq), -(-N // bkv)
    ws = torch.zeros(sla.sla_workspace_size(shape, mode), dtype=torch.uint8, device=dev)
    kept = torch.full((B, H, nq, k_keep), -7, dtype=torch.int32, device=dev)
    labels = torch.full((B, H, nq, nkv), 9, dtype=torch.int8, device=dev)
    scores = torch.full((B, H, nq, nkv), float("nan"), dtype=torch.float32, device=dev)
    sla.sla_route(shape, qd, kd, None if wq is None else wq.to(dev), None if wk is None else wk.to(dev), mode,
                  k_keep, k_neg, kept, labels, scores, ws)
    assert sla.sla_read_device_status(ws) == 0
    return kept.cpu().numpy(), labels.cpu().numpy(), scores.cpu().numpy()


def run_route_after_prepare(q, k, v, wq, wk, bq, bkv, mode, k_keep, k_neg=0):
    """sla_prepare, then sla_route with SLA_ROUTE_KBAR_FROM_WS (key-block means
    from the prepass) on the same workspace."""
    dev = "cuda"
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    shape = sla.make_shape(qd, bq, bkv)
    B, H, N, d = q.shape
    nq, nkv = -(-N // bq), -(-N // bkv)
    ws = torch.zeros(sla.sla_workspace_size(shape, mode), dtype=torch.uint8, device=dev)
    kept = torch.full((B, H, nq, k_keep), -7, dtype=torch.int32, device=dev)
    labels = torch.full((B, H, nq, nkv), 9, dtype=torch.int8, device=dev)
    scores = torch.full((B, H, nq, nkv), float("nan"), dtype=torch.float32, device=dev)
    sla.sla_prepare(shape, kd, vd, sla.SLA_PHI_ELU1, ws)
    sla.sla_route(shape, qd, kd, None if wq is None else wq.to(dev), None if wk is None else wk.to(dev),
                  mode | sla.SLA_ROUTE_KBAR_FROM_WS, k_keep, k_neg, kept, labels, scores, ws)
    assert sla.sla_read_device_status(ws) == 0
    return kept.cpu().numpy(), labels.cpu().numpy(), scores.cpu().numpy()


def run_route_soft(q, k, wq, wk, bq, bkv, k_keep, tau):
    """sla_route_soft through the C ABI: (mask [B,H,n_q,n_kv], lambda [B,H,n_q])."""
    dev = "cuda"
    qd, kd = q.to(dev), k.to(dev)
    shape = sla.make_shape(qd, bq, bkv)
    B, H, N, d = q.shape
    nq, nkv = -(-N // bq), -(-N // bkv)
    ws = torch.zeros(sla.sla_workspace_size(shape, 0), dtype=torch.uint8, device=dev)
    mask = torch.full((B, H, nq, nkv), float("nan"), dtype=torch.float32, device=dev)
    lam = torch.full((B, H, nq), float("nan"), dtype=torch.float32, device=dev)
    sla.sla_route_soft(shape, qd, kd, None if wq is None else wq.to(dev), None if wk is None else wk.to(dev),
                       k_keep, tau, mask, lam, ws)
    assert sla.sla_read_device_status(ws) == 0
    return mask.cpu().numpy(), lam.cpu().numpy()


def run_sla2(q, k, v, kept, alpha, bq, bkv, phi=sla.SLA_PHI_ELU1, out_dtype=torch.float32, flags=0, ws=None):
    dev = "cuda"
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    shape = sla.make_shape(qd, bq, bkv)
    if ws is None:
        mode = sla.SLA_WS_FP8 if flags & (sla.SLA_FLAG_FP8 | sla.SLA_FLAG_INT8) else 0
        ws = torch.zeros(sla.sla_workspace_size(shape, mode), dtype=torch.uint8, device=dev)
    kt = torch.as_tensor(np.ascontiguousarray(kept), dtype=torch.int32).to(dev)
    out = torch.full(q.shape, float("nan"), dtype=out_dtype, device=dev)
    sla.sla2_attn_fwd(shape, qd, kd, vd, kt, int(kept.shape[-1]), alpha.to(dev).contiguous(), phi, flags, out, ws)
    assert sla.sla_read_device_status(ws) == 0
    return out.float().cpu().numpy()


def run_sla(q, k, v, labels, wproj, bq, bkv, phi=sla.SLA_PHI_ELU1, out_dtype=torch.float32):
    dev = "cuda"
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    shape = sla.make_shape(qd, bq, bkv)
    ws = torch.zeros(sla.sla_workspace_size(shape, 1), dtype=torch.uint8, device=dev)
    lab = torch.as_tensor(np.ascontiguousarray(labels), dtype=torch.int8).to(dev)
    out = torch.full(q.shape, float("nan"), dtype=out_dtype, device=dev)
    sla.sla_attn_fwd(shape, qd, kd, vd, lab, wproj.to(dev).contiguous(), phi, 0, out, ws)
    assert sla.sla_read_device_status(ws) == 0
    return out.float().cpu().numpy()


def rows_of(blocks, bq, N):
    return [(b, h, np.arange(i * bq, min((i + 1) * bq, N))) for (b, h, i) in blocks]


def compare(got, want, blocks, bq, tol=TOL_BF16, rel_l1=TOL_REL_L1):
    """Max-abs and relative-L1 error of got vs want over the rows of `blocks`."""
    N = got.shape[2]
    g = np.concatenate([got[b, h, r] for b, h, r in rows_of(blocks, bq, N)])
    w = np.concatenate([want[b, h, r] for b, h, r in rows_of(blocks, bq, N)])
    assert np.isfinite(g).all(), "non-finite output"
    err = np.abs(g - w)
    mx = float(err.max())
    rl1 = float(err.sum() / max(np.abs(w).sum(), 1e-30))
    assert mx <= tol, f"max-abs {mx:.3e} > {tol:.1e} (rel-L1 {rl1:.2e})"
    assert rl1 <= rel_l1, f"rel-L1 {rl1:.3e} > {rel_l1:.1e}"
    return mx, rl1


def sample_blocks(B, H, nq, per_head=4, seed=0):
    rng = np.random.default_rng(seed)
    out = []
    for b in range(B):
        for h in range(H):
            picks = {0, nq - 1} | set(int(x) for x in rng.integers(0, nq, per_head - 2))
            out += [(b, h, i) for i in sorted(picks)]
    return out
