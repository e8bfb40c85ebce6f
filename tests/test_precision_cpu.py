"""Why the attention kernel stages P (and with it V, phi(K)) in fp16: at the
Wan2.1-1.3B shape, rounding P to bf16 before P.V moves the sparse branch's
output by about the 2e-3 max-abs gate, fp16 by a tenth of it.

"SLA2: Sparse-Linear Attention with Learnable Routing and QAT" §2.B (P.V on
the kept blocks) with everything but the rounding of P in fp64; the kept
blocks come from the oracle's router on the seeded workload."""
import math

import numpy as np
import torch

from oracle import sla_oracle as orc
from sparse_linear_attention_b200 import inputs


def _p_rounding_errors(heads, blocks_per_head, seed=0):
    w = inputs.WORKLOADS["wan13"]
    x = inputs.make_inputs(w, heads=heads)
    errs = {torch.float16: 0.0, torch.bfloat16: 0.0}
    rng = np.random.default_rng(seed)
    for h in heads:
        q = x["q"][:, h:h + 1].float().numpy()
        k = x["k"][:, h:h + 1].float().numpy()
        kept, _, _ = orc.route(q, k, x["wq"].numpy(), x["wk"].numpy(), w.bq, w.bkv, "sla2", orc.keep_count(w.keep_ratio, w.n_kv))
        qd, kd, vd = (t[0, h].double().numpy() for t in (x["q"], x["k"], x["v"]))
        for i in rng.choice(w.n_q, blocks_per_head, replace=False):
            rows = np.arange(i * w.bq, min((i + 1) * w.bq, w.N))
            keys = np.concatenate([np.arange(j * w.bkv, min((j + 1) * w.bkv, w.N)) for j in kept[0, 0, i]])
            s = qd[rows] @ kd[keys].T / math.sqrt(w.d)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            l = p.sum(axis=1, keepdims=True)
            o = p @ vd[keys] / l
            for dt in errs:
                pr = torch.from_numpy(p).to(dt).double().numpy()
                errs[dt] = max(errs[dt], float(np.abs(pr @ vd[keys] / l - o).max()))
    return errs


def test_bf16_p_reaches_the_gate_and_fp16_p_does_not():
    errs = _p_rounding_errors(heads=[0, 5], blocks_per_head=6)
    assert errs[torch.float16] < 1e-3
    assert errs[torch.bfloat16] > 1.5e-3
    assert errs[torch.bfloat16] > 4 * errs[torch.float16]
