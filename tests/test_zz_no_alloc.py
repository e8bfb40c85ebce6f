"""The workspace-free router entry point (sla_route_noalloc) on a B200.

It serves callers that cannot give the library device memory where they
route (code under another framework's memory manager, or code that must not
call cudaMalloc there).  Its scratch is a fixed array inside libsla, shared by
all calls.  This test calls it through the C ABI three times in a row, on different
inputs, so each call after the first starts from the previous call's leftover
scratch (the last one with a key count that is not a multiple of four, so
stale padding columns are read and must be dropped), and checks each result
against sla_route with a caller-owned workspace.  Router
results are compared bit for bit, as in the other router tests.  The file is
named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_linear_attention_b200 import inputs, sla

pytestmark = pytest.mark.gpu


def _route_both(w, x, mode, k_keep, k_neg):
    dev = "cuda"
    q, k = x["q"].to(dev), x["k"].to(dev)
    wq, wk = x["wq"].to(dev), x["wk"].to(dev)
    shape = sla.make_shape(q, w.bq, w.bkv)
    nq, nkv = w.n_q, w.n_kv
    outs = []
    for use_ws in (True, False):
        kept = torch.full((w.B, w.H, nq, k_keep), -5, dtype=torch.int32, device=dev)
        labels = torch.full((w.B, w.H, nq, nkv), 7, dtype=torch.int8, device=dev)
        scores = torch.full((w.B, w.H, nq, nkv), float("nan"), dtype=torch.float32, device=dev)
        if use_ws:
            ws = torch.zeros(sla.sla_workspace_size(shape, mode), dtype=torch.uint8, device=dev)
            sla.sla_route(shape, q, k, wq, wk, mode, k_keep, k_neg, kept, labels, scores, ws)
        else:
            st = sla.lib().sla_route_noalloc(ctypes.byref(shape), ctypes.c_void_p(q.data_ptr()),
                                             ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(wq.data_ptr()),
                                             ctypes.c_void_p(wk.data_ptr()), mode, k_keep, k_neg,
                                             ctypes.c_void_p(kept.data_ptr()), ctypes.c_void_p(labels.data_ptr()),
                                             ctypes.c_void_p(scores.data_ptr()),
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
            assert st == sla.SLA_OK, sla.lib().sla_last_error_detail().decode()
        torch.cuda.synchronize()
        outs.append((kept.cpu().numpy(), labels.cpu().numpy(), scores.cpu().numpy()))
    return outs


def test_noalloc_router_matches_workspace_router_on_two_calls():
    big = inputs.WORKLOADS["wan13"]
    tiny = inputs.WORKLOADS["tiny"]
    # n_kv = 15: the key-mean rows are padded to 16 columns, and the padding
    # column keeps what the larger calls before it left in the shared scratch
    ragged = inputs.Workload("ragged", 1, 3, (1, 1, 900), 128, 128, 64, "bf16", keep_count=3)
    cases = [
        (big, inputs.make_inputs(big), sla.SLA_MODE_SLA2_TOPK, sla.sla_keep_count(0.03, big.n_kv), 0),
        (tiny, inputs.make_inputs(tiny), sla.SLA_MODE_SLA_3WAY, 3, 2),
        (ragged, inputs.random_inputs(1, 3, 900, 128, dtype="bf16", seed=21, scale=1.5, n_q=ragged.n_q),
         sla.SLA_MODE_SLA2_TOPK, 3, 0),
    ]
    assert ragged.n_kv % 4 != 0
    for w, x, mode, kk, kn in cases:  # calls in a row, different shapes and inputs
        (k1, l1, s1), (k2, l2, s2) = _route_both(w, x, mode, kk, kn)
        assert np.array_equal(s1.view(np.uint32), s2.view(np.uint32)), w.name
        assert np.array_equal(k1, k2), w.name
        assert np.array_equal(l1, l2), w.name


def test_noalloc_router_rejects_shapes_beyond_its_scratch():
    w = inputs.WORKLOADS["wan14"]  # needs ~36 MB of router scratch
    shape = sla.Shape(w.B, w.H, w.N, w.d, w.bq, w.bkv, sla.SLA_BF16)
    fake = ctypes.c_void_p(1 << 40)  # never touched: the size check fails first
    st = sla.lib().sla_route_noalloc(ctypes.byref(shape), fake, fake, None, None, 0, 35, 0, fake, None, None, None)
    assert sla.STATUS_NAMES[st] == "SLA_ERR_WORKSPACE"
    assert "16777216" in sla.lib().sla_last_error_detail().decode()
