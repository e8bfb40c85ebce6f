"""libsla's C ABI on the host (no GPU): every symbol in include/sla.h is
exported, and argument checks fail before anything is launched."""
import ctypes
import os
import re
import subprocess

import pytest

from oracle import sla_oracle
from sparse_linear_attention_b200 import sla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "sla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sla\w+)\s*\(", src)))


def test_header_matches_binding():
    assert _header_functions() == sorted(sla.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = sla.lib()
    out = subprocess.run(["nm", "-D", "--defined-only", sla.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (\w+)$", out, flags=re.M))
    for name in _header_functions():
        assert name in exported, name
        assert hasattr(L, name)


def test_status_strings():
    for code, name in sla.STATUS_NAMES.items():
        assert sla.lib().sla_status_string(code).decode() == name


@pytest.mark.parametrize("n_kv", [1, 7, 16, 512, 591, 1182, 2048])
def test_keep_count_matches_oracle(n_kv):
    for ratio in [0.0, 1e-6, 0.01, 0.03, 0.04, 0.05, 0.1, 0.25, 0.5, 0.97, 1.0, 1.5]:
        assert sla.sla_keep_count(ratio, n_kv) == sla_oracle.keep_count(ratio, n_kv), (ratio, n_kv)


def _shape(**kw):
    base = dict(B=1, H=12, N=32760, d=128, bq=128, bkv=64, in_dtype=sla.SLA_BF16)
    base.update(kw)
    return sla.Shape(**base)


def test_workspace_size():
    good = _shape()
    a = sla.sla_workspace_size(good, sla.SLA_MODE_SLA2_TOPK)
    b = sla.sla_workspace_size(good, sla.SLA_MODE_SLA_3WAY)
    assert 0 < a < b
    assert a % 256 == 0
    # phi(K) and V staged as fp16 [BH, N, 128] dominate
    assert a >= 2 * 12 * 32760 * 128 * 2
    for bad in [dict(d=100), dict(d=136), dict(bq=96), dict(bkv=128), dict(N=0), dict(N=131073),
                dict(B=0), dict(in_dtype=7)]:
        assert sla.sla_workspace_size(_shape(**bad), 0) == 0, bad
    assert sla.sla_workspace_size(good, 5) == 0
    # f32 inputs or d != 128 need the padded bf16 copies of Q and K
    assert sla.sla_workspace_size(_shape(d=64), 0) > sla.sla_workspace_size(_shape(), 0) // 2


FAKE = 0x7F0000000000  # never dereferenced: every call below fails its checks first


def _route(shape, q=FAKE, k=FAKE, mode=0, k_keep=15, k_neg=0, kept=FAKE, ws=FAKE, ws_bytes=1 << 40, wq=None):
    return sla.lib().sla_route(ctypes.byref(shape), q, k, wq, None, mode, k_keep, k_neg, kept, None, None,
                               ws, ws_bytes, None)


def test_route_rejects_bad_arguments_before_launch():
    s = _shape()
    assert _route(s, q=None) == 1
    assert _route(s, q=FAKE + 2) == 3
    assert _route(s, wq=FAKE + 4) == 3       # projections are read 16 bytes at a time
    assert _route(s, mode=3) == 1
    assert _route(s, k_keep=513) == 1
    assert _route(s, k_keep=-1) == 1
    assert _route(s, k_neg=1) == 1            # SLA2 takes no negligible count
    assert _route(s, mode=1, k_keep=300, k_neg=300) == 1
    assert _route(s, kept=None) == 1
    assert _route(s, ws=None) == 1
    assert _route(s, ws=FAKE + 16) == 3       # workspace must be 256-byte aligned
    assert _route(s, ws_bytes=1000) == 4
    assert _route(_shape(N=131072 + 64)) == 2
    assert _route(s, kept=None) == 1
    assert "kept_idx" in sla.lib().sla_last_error_detail().decode()


def test_route_key_means_flag_checks():
    """SLA_ROUTE_KBAR_FROM_WS (key-block means from the prepass) exists only
    where the prepass writes them: bf16 inputs with d = 128."""
    flag = sla.SLA_ROUTE_KBAR_FROM_WS
    assert _route(_shape(d=64), mode=flag) == 2
    assert _route(_shape(in_dtype=sla.SLA_F32), mode=flag) == 2
    assert "d = 128" in sla.lib().sla_last_error_detail().decode()
    assert _route(_shape(), mode=flag | 3) == 1       # the base mode is still checked
    assert _route(_shape(), mode=flag, kept=None) == 1  # and the other arguments
    # the route without a workspace takes no flag
    L = sla.lib()
    assert L.sla_route_noalloc(ctypes.byref(_shape()), FAKE, FAKE, None, None, flag, 15, 0, FAKE, None, None,
                               None) == 1


def test_route_soft_rejects_bad_arguments_before_launch():
    s = _shape()
    L = sla.lib()

    def call(**kw):
        a = dict(q=FAKE, k=FAKE, wq=None, k_keep=15, tau=0.1, mask=FAKE, lam=None, ws=FAKE, wsb=1 << 40)
        a.update(kw)
        return L.sla_route_soft(ctypes.byref(a.pop("shape", s)), a["q"], a["k"], a["wq"], None, a["k_keep"],
                                a["tau"], a["mask"], a["lam"], a["ws"], a["wsb"], None)

    assert call(q=None) == 1
    assert call(mask=None) == 1
    assert "mask" in L.sla_last_error_detail().decode()
    for tau in (0.0, -0.1, float("inf"), float("nan")):
        assert call(tau=tau) == 1, tau
    assert call(k_keep=-1) == 1
    assert call(k_keep=513) == 1
    assert call(q=FAKE + 8) == 3
    assert call(wq=FAKE + 4) == 3
    assert call(ws=None) == 1
    assert call(wsb=1000) == 4
    assert call(shape=_shape(N=131072 + 64)) == 2


def test_attention_rejects_bad_arguments_before_launch():
    s = _shape()
    L = sla.lib()

    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, kept=FAKE, k_keep=15, alpha=FAKE, phi=0, flags=0, out=FAKE, odt=1,
                 ws=FAKE, wsb=1 << 40)
        a.update(kw)
        return L.sla2_attn_fwd(ctypes.byref(s), a["q"], a["k"], a["v"], a["kept"], a["k_keep"], a["alpha"],
                               a["phi"], a["flags"], a["out"], a["odt"], a["ws"], a["wsb"], None)

    assert call(v=None) == 1
    assert call(k=FAKE + 8) == 3
    assert call(k_keep=513) == 1
    assert call(kept=None) == 1
    assert call(alpha=None) == 1
    assert call(phi=2) == 1
    assert call(flags=16) == 1
    assert call(flags=sla.SLA_FLAG_FP8 | sla.SLA_FLAG_INT8) == 1  # the two low-bit formats exclude each other
    assert "exclude" in L.sla_last_error_detail().decode()
    # the low-bit branches need the larger workspace (sla_workspace_size with SLA_WS_FP8)
    need = sla.sla_workspace_size(s, 0)
    assert call(flags=sla.SLA_FLAG_FP8, wsb=need) == 4
    assert call(flags=sla.SLA_FLAG_INT8, wsb=need) == 4
    assert call(out=None) == 1
    assert call(out=FAKE + 4) == 3
    assert call(odt=9) == 1
    assert call(wsb=10) == 4
    assert "ws" in L.sla_last_error_detail().decode()

    def call3(**kw):
        a = dict(labels=FAKE, wp=FAKE, wsb=1 << 40)
        a.update(kw)
        return L.sla_attn_fwd(ctypes.byref(s), FAKE, FAKE, FAKE, a["labels"], a["wp"], 0, 0, FAKE, 1, FAKE,
                              a["wsb"], None)

    assert call3(labels=None) == 1
    assert call3(wp=None) == 1
    assert call3(wp=FAKE + 2) == 3
    for low in (sla.SLA_FLAG_FP8, sla.SLA_FLAG_INT8):  # the low-bit branches: SLA2 only
        assert L.sla_attn_fwd(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, 0, low, FAKE, 1, FAKE,
                              1 << 40, None) == 2
    # the SLA workspace also holds the per-row block lists
    need2 = sla.sla_workspace_size(s, 0)
    assert call3(wsb=need2) == 4


def test_prepare_rejects_bad_arguments_before_launch():
    s = _shape()
    L = sla.lib()
    assert L.sla_prepare(ctypes.byref(s), None, FAKE, 0, FAKE, 1 << 40, None) == 1
    assert L.sla_prepare(ctypes.byref(s), FAKE, FAKE, 5, FAKE, 1 << 40, None) == 1
    assert L.sla_prepare(ctypes.byref(_shape(bkv=32)), FAKE, FAKE, 0, FAKE, 1 << 40, None) == 2


def test_backward_rejects_bad_arguments_before_launch():
    s = _shape()
    L = sla.lib()
    need = sla.sla2_attn_bwd_workspace_size(s)
    # status + H_tot, Z_tot and their gradients + the [BH, N, 128] fp32 key-side sums
    assert need >= 12 * 32760 * 128 * 4 and need % 256 == 0
    assert sla.sla2_attn_bwd_workspace_size(_shape(d=100)) == 0

    def call(**kw):
        a = dict(q=FAKE, kept=FAKE, k_keep=15, alpha=FAKE, phi=0, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE,
                 dal=FAKE, ws=FAKE, wsb=need)
        a.update(kw)
        return L.sla2_attn_bwd(ctypes.byref(s), a["q"], FAKE, FAKE, a["kept"], a["k_keep"], a["alpha"], a["phi"],
                               a["dout"], a["dq"], a["dk"], a["dv"], a["dal"], a["ws"], a["wsb"], None)

    assert call(q=None) == 1
    assert call(q=FAKE + 2) == 3
    assert call(k_keep=-1) == 1
    assert call(k_keep=513) == 1
    assert call(kept=None) == 1
    assert call(alpha=None) == 1
    assert call(phi=3) == 1
    for name in ("dout", "dq", "dk", "dv", "dal"):
        assert call(**{name: None}) == 1, name
        assert call(**{name: FAKE + 4}) == 3, name
    assert call(ws=None) == 1
    assert call(ws=FAKE + 16) == 3
    assert call(wsb=need - 1) == 4
    assert "sla2_attn_bwd_workspace_size" in L.sla_last_error_detail().decode()
    assert L.sla2_attn_bwd(ctypes.byref(_shape(bq=96)), FAKE, FAKE, FAKE, FAKE, 15, FAKE, 0, FAKE, FAKE, FAKE,
                           FAKE, FAKE, FAKE, need, None) == 2


def test_backward_workspace_layout():
    """CUDA-core path: status word, H_tot and Z_tot, their gradients, and the
    [BH, N, 128] fp32 key-side buffer, each rounded up to 256 bytes.
    Tensor-core path (bf16, d = 128, b_q = 128): the forward's SLA2 workspace,
    then the per-row statistics, phi(Q) in fp16, the inverse block lists, the
    dH (fp16) / dZ partials per query tile, dH_tot, dZ_tot, and the fp16 copy
    of dH_tot with its per-head scale."""
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    for B, H, N, d, dt in [(1, 12, 32760, 64, sla.SLA_BF16), (2, 3, 1000, 64, sla.SLA_BF16), (1, 1, 1, 8, sla.SLA_F32),
                           (1, 40, 75600, 128, sla.SLA_F32)]:
        s = _shape(B=B, H=H, N=N, d=d, in_dtype=dt)
        BH = B * H
        want = 256 + 2 * (a256(BH * 128 * 128 * 4) + a256(BH * 128 * 4)) + a256(BH * N * 128 * 4)
        assert sla.sla2_attn_bwd_workspace_size(s) == want, (B, H, N, d)
    for B, H, N in [(1, 12, 32760), (2, 3, 1000), (1, 1, 1), (1, 40, 75600)]:
        s = _shape(B=B, H=H, N=N, d=128, bq=128, in_dtype=sla.SLA_BF16)
        BH, nq, nkv = B * H, -(-N // 128), -(-N // 64)
        want = (sla.sla_workspace_size(s, sla.SLA_MODE_SLA2_TOPK) + a256(BH * N * 32) + a256(BH * N * 256)
                + a256(BH * nkv * nq * 4) + a256(BH * nkv * 4) + a256(BH * nq * 32768) + a256(BH * nq * 512)
                + a256(BH * 65536) + a256(BH * 512) + a256(BH * 32768) + a256(BH * 4))
        assert sla.sla2_attn_bwd_workspace_size(s) == want, (B, H, N)


def test_sla_backward_rejects_bad_arguments_before_launch():
    s = _shape()
    L = sla.lib()
    need = sla.sla_attn_bwd_workspace_size(s)
    # the key-side buffer and the O_l rows, both fp32 [BH, N, 128], among the rest
    assert need >= 2 * 12 * 32760 * 128 * 4 and need % 256 == 0
    assert sla.sla_attn_bwd_workspace_size(_shape(d=100)) == 0

    def call(**kw):
        a = dict(q=FAKE, labels=FAKE, wp=FAKE, phi=0, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, dwp=FAKE, ws=FAKE,
                 wsb=need)
        a.update(kw)
        return L.sla_attn_bwd(ctypes.byref(s), a["q"], FAKE, FAKE, a["labels"], a["wp"], a["phi"], a["dout"],
                              a["dq"], a["dk"], a["dv"], a["dwp"], a["ws"], a["wsb"], None)

    assert call(q=None) == 1
    assert call(labels=None) == 1
    assert call(wp=None) == 1
    assert call(phi=2) == 1
    for name in ("dout", "dq", "dk", "dv"):
        assert call(**{name: None}) == 1, name
        assert call(**{name: FAKE + 4}) == 3, name
    assert call(dwp=None) == 1
    assert call(ws=None) == 1
    assert call(ws=FAKE + 16) == 3
    assert call(wsb=need - 1) == 4
    assert "sla_attn_bwd_workspace_size" in L.sla_last_error_detail().decode()


def test_sla_backward_workspace_layout():
    """The CUDA-core backward's workspace, then the critical / negligible lists and
    their counts, the [BH, N, 128] fp32 O_l rows and the dW_proj partials of
    about two row splits per SM, each rounded up to 256 bytes."""
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    for B, H, N, d, bq in [(1, 12, 32760, 128, 128), (2, 3, 1000, 64, 64), (1, 1, 1, 8, 64)]:
        s = _shape(B=B, H=H, N=N, d=d, bq=bq)
        BH, nq, nkv = B * H, -(-N // bq), -(-N // 64)
        rows = BH * N
        per = max(32, -(-(-(-rows // 296)) // 32) * 32)
        nsplit = -(-rows // per)
        fp32_ws = 256 + 2 * (a256(BH * 128 * 128 * 4) + a256(BH * 128 * 4)) + a256(BH * N * 128 * 4)
        want = (fp32_ws + a256(BH * nq * 2 * nkv * 4) + a256(BH * nq * 2 * 4) + a256(rows * 128 * 4)
                + a256(nsplit * 128 * 128 * 4))
        assert sla.sla_attn_bwd_workspace_size(s) == want, (B, H, N, d)


def _noalloc(shape, q=FAKE, k=FAKE, mode=0, k_keep=15, k_neg=0, kept=FAKE, wq=None):
    L = sla.lib()
    sp = ctypes.byref(shape) if shape is not None else None
    st = L.sla_route_noalloc(sp, q, k, wq, None, mode, k_keep, k_neg, kept, None, None, None)
    return st, L.sla_last_error_detail().decode()


def test_route_noalloc_rejects_with_a_detail_naming_the_argument():
    """Every early reject of the workspace-free router replaces the thread's
    last error detail with one naming the rejected argument (and none of these
    calls reaches the GPU)."""
    s = _shape()
    cases = [
        (dict(shape=None), 1, "shape is null"),
        (dict(shape=_shape(d=100)), 2, "d must be"),
        (dict(shape=_shape(bq=96)), 2, "bq"),
        (dict(shape=_shape(B=0)), 1, "positive"),
        (dict(shape=s, mode=sla.SLA_MODE_SLA2_TOPK | sla.SLA_ROUTE_KBAR_FROM_WS), 1, "SLA_ROUTE_KBAR_FROM_WS"),
        (dict(shape=s, mode=9), 1, "mode"),
        (dict(shape=s, q=None), 1, "Q or K is null"),
        (dict(shape=s, k=FAKE + 8), 3, "16-byte"),
        (dict(shape=s, wq=FAKE + 4), 3, "Wq, Wk"),
        (dict(shape=s, k_keep=600), 1, "k_keep"),
        (dict(shape=s, k_neg=2), 1, "k_neg"),
        (dict(shape=s, kept=None), 1, "kept_idx"),
    ]
    for kw, code, words in cases:
        # a different failure first, so a stale detail would show
        _route(_shape(), q=None)
        st, detail = _noalloc(**kw)
        assert st == code, (kw, st, detail)
        assert words in detail and detail.startswith("sla_route_noalloc"), (kw, detail)


def test_binding_refuses_host_tensors():
    """The binding checks where each tensor lives before passing its pointer:
    a CPU tensor never reaches the C side as a device pointer."""
    import torch
    q = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16)
    shape = sla.make_shape(q, 64)
    ws = torch.zeros(256, dtype=torch.uint8)
    kept = torch.zeros(1, 2, 1, 1, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        sla.sla_route(shape, q, q, None, None, 0, 1, 0, kept, None, None, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        sla.sla_prepare(shape, q, q, 0, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        sla.sla2_attn_fwd(shape, q, q, q, kept, 1, torch.zeros(1, 2, 1), 0, 0, torch.zeros_like(q), ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        sla.sla_read_device_status(ws)
    g = torch.zeros(1, 2, 64, 64)
    with pytest.raises(ValueError, match="CUDA tensor"):
        sla.sla2_attn_bwd(shape, q, q, q, kept, 1, torch.zeros(1, 2, 1), 0, q, g, g, g, torch.zeros(1, 2, 1), ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        sla.sla_attn_bwd(shape, q, q, q, torch.zeros(1, 2, 1, 1, dtype=torch.int8),
                         torch.zeros(64, 64, dtype=torch.bfloat16), 0, q, g, g, g, torch.zeros(64, 64), ws)
    with pytest.raises(TypeError):
        sla.sla_route(shape, "q", q, None, None, 0, 1, 0, kept, None, None, ws)
