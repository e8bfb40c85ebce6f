"""Seeded synthetic workloads for SLA2 / SLA attention forward.

This module only draws inputs. It holds none of the attention arithmetic, so the
CPU oracle (tests) and the CUDA path (library) can both be fed from it without
sharing any of the method's code.

Stand-in for Wan2.1 video attention activations (no model weights or videos are
available): per (batch, head) a smooth low-frequency field G over the
(frames x height x width) latent grid is shared by Q and K, V gets its own field,
and each tensor adds i.i.d. N(0,1) noise:

    G(t,y,x)[c] = sum_{m<16} a[m,c] * cos(2*pi*(ft_m*t/T + fy_m*y/Hg + fx_m*x/Wg) + psi_m)
    ft, fy, fx ~ U{0..3},  psi ~ U(0, 2*pi),  a ~ N(0, 1/16)
    Q = s*(G + eps_q),  K = s*(G + eps_k),  V = Gv + eps_v

Token n sits at grid position n = (t*Hg + y)*Wg + x.  The scale s sharpens
softmax rows (s^2 = 16/sqrt(d) for the video-shaped workloads, 1 for the tiny
one).  Router weights W_q, W_k ~ N(0, 1/d) (fp32, d x d, shared by all heads),
the SLA2 mixing ratio alpha = sigmoid(N(0,1)) per (batch, head, query block), and
the SLA output projection W_proj ~ N(0, 1/d) rounded to bf16.

Each (batch, head) draws from its own torch CPU generator seeded from
(seed, b, h), so any subset of heads is reproducible on its own.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    grid: tuple  # (T, Hg, Wg) latent grid; N = T*Hg*Wg
    d: int
    bq: int
    bkv: int
    dtype: str  # "f32" or "bf16": storage type of Q, K, V
    keep_ratio: float = 0.03  # SLA2: fraction of KV blocks kept per query block
    keep_count: int | None = None  # explicit count overrides keep_ratio
    mode: str = "sla2"  # "sla2" (top-k + alpha mix) or "sla" (3-way labels + proj)
    crit_ratio: float = 0.05  # SLA: critical fraction k_h
    negl_ratio: float = 0.10  # SLA: negligible fraction k_l
    fp8: bool = False
    scale: float | None = None  # s; default 1 for f32, (16/sqrt(d))**0.5 otherwise
    seed: int = 0

    @property
    def N(self) -> int:
        T, Hg, Wg = self.grid
        return T * Hg * Wg

    @property
    def n_q(self) -> int:
        return -(-self.N // self.bq)

    @property
    def n_kv(self) -> int:
        return -(-self.N // self.bkv)

    @property
    def s(self) -> float:
        if self.scale is not None:
            return self.scale
        return 1.0 if self.dtype == "f32" else (16.0 / math.sqrt(self.d)) ** 0.5


# The named workloads.  "tiny" is small enough for the pure-numpy oracle to
# finish in seconds; the others carry the Wan2.1 latent shapes.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, (4, 16, 16), 64, 64, 64, "f32", keep_count=4, seed=0),
    "wan13": Workload("wan13", 1, 12, (21, 30, 52), 128, 128, 64, "bf16", keep_ratio=0.03, seed=1),
    "sla13": Workload("sla13", 1, 12, (21, 30, 52), 128, 128, 64, "bf16", mode="sla",
                      crit_ratio=0.05, negl_ratio=0.10, seed=1),
    # SLA with the block sizes of its own page (64 x 64)
    "sla13_64": Workload("sla13_64", 1, 12, (21, 30, 52), 128, 64, 64, "bf16", mode="sla",
                         crit_ratio=0.05, negl_ratio=0.10, seed=1),
    "wan14": Workload("wan14", 1, 40, (21, 45, 80), 128, 128, 64, "bf16", keep_ratio=0.03, seed=2),
    "fp8_13": Workload("fp8_13", 1, 12, (21, 30, 52), 128, 128, 64, "bf16", keep_ratio=0.03, fp8=True, seed=1),
    "fp8_14": Workload("fp8_14", 1, 40, (21, 45, 80), 128, 128, 64, "bf16", keep_ratio=0.03,
                       fp8=True, seed=2),
}


def _head_generator(seed: int, b: int, h: int, stream: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(((seed * 1000003 + b) * 1009 + h) * 17 + stream)
    return g


def _field(g: torch.Generator, grid, d: int) -> torch.Tensor:
    """Smooth low-frequency field on the latent grid, [N, d] float64."""
    T, Hg, Wg = grid
    m = 16
    f = torch.randint(0, 4, (m, 3), generator=g, dtype=torch.int64).to(torch.float64)
    psi = torch.rand(m, generator=g, dtype=torch.float64) * (2 * math.pi)
    a = torch.randn(m, d, generator=g, dtype=torch.float64) / 4.0  # std 1/4 -> var 1/16
    t = torch.arange(T, dtype=torch.float64).view(T, 1, 1) / T
    y = torch.arange(Hg, dtype=torch.float64).view(1, Hg, 1) / Hg
    x = torch.arange(Wg, dtype=torch.float64).view(1, 1, Wg) / Wg
    ph = (2 * math.pi) * (f[:, 0].view(m, 1, 1, 1) * t + f[:, 1].view(m, 1, 1, 1) * y
                          + f[:, 2].view(m, 1, 1, 1) * x) + psi.view(m, 1, 1, 1)
    basis = torch.cos(ph).reshape(m, T * Hg * Wg)  # [m, N]
    return basis.t() @ a  # [N, d]


def _store(x: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return x.to(torch.bfloat16)
    # f32 workloads hold values on the bf16 grid, so the tensor-core operands
    # (bf16) represent them exactly; the storage type stays float32.
    return x.to(torch.bfloat16).to(torch.float32)


def make_inputs(w: Workload, heads=None) -> dict:
    """Draw Q, K, V [B,H,N,d] plus router/mixing parameters for workload w.

    heads: optional list of head indices to draw (others are left zero); all
    heads by default.  Returns CPU tensors.
    """
    B, H, N, d = w.B, w.H, w.N, w.d
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q = torch.zeros(B, H, N, d, dtype=tdt)
    k = torch.zeros(B, H, N, d, dtype=tdt)
    v = torch.zeros(B, H, N, d, dtype=tdt)
    alpha = torch.zeros(B, H, w.n_q, dtype=torch.float32)
    hs = range(H) if heads is None else heads
    s = w.s
    for b in range(B):
        for h in hs:
            g = _head_generator(w.seed, b, h, 0)
            G = _field(g, w.grid, d)
            Gv = _field(g, w.grid, d)
            eq = torch.randn(N, d, generator=g, dtype=torch.float32).to(torch.float64)
            ek = torch.randn(N, d, generator=g, dtype=torch.float32).to(torch.float64)
            ev = torch.randn(N, d, generator=g, dtype=torch.float32).to(torch.float64)
            q[b, h] = _store(s * (G + eq), w.dtype)
            k[b, h] = _store(s * (G + ek), w.dtype)
            v[b, h] = _store(Gv + ev, w.dtype)
            alpha[b, h] = torch.sigmoid(torch.randn(w.n_q, generator=g, dtype=torch.float32))
    gw = _head_generator(w.seed, 0, 0, 1)
    wq = (torch.randn(d, d, generator=gw, dtype=torch.float32) / math.sqrt(d)).contiguous()
    wk = (torch.randn(d, d, generator=gw, dtype=torch.float32) / math.sqrt(d)).contiguous()
    wproj = (torch.randn(d, d, generator=gw, dtype=torch.float32) / math.sqrt(d)).to(torch.bfloat16)
    return {"q": q, "k": k, "v": v, "wq": wq, "wk": wk, "alpha": alpha, "wproj": wproj}


def random_inputs(B, H, N, d, dtype="bf16", seed=0, scale=1.0, n_q=1):
    """Plain N(0, scale^2) Q, K, V for edge-case tests (ragged N, odd sizes)."""
    g = torch.Generator()
    g.manual_seed(seed)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = {}
    for name in ("q", "k", "v"):
        x = torch.randn(B, H, N, d, generator=g, dtype=torch.float32) * scale
        out[name] = _store(x, dtype) if dtype == "f32" else x.to(tdt)
    out["alpha"] = torch.sigmoid(torch.randn(B, H, n_q, generator=g, dtype=torch.float32))
    out["wq"] = torch.randn(d, d, generator=g, dtype=torch.float32) / math.sqrt(d)
    out["wk"] = torch.randn(d, d, generator=g, dtype=torch.float32) / math.sqrt(d)
    out["wproj"] = (torch.randn(d, d, generator=g, dtype=torch.float32) / math.sqrt(d)).to(torch.bfloat16)
    return out
