"""bench.py's work counts on the CPU: the algorithmic work its roofline and
effective-TOPS figures divide by, against a brute-force count."""
import numpy as np
import torch

import bench
from sparse_linear_attention_b200 import inputs


def _brute(w, kept):
    """4 d per (query row, kept valid key), counted token by token."""
    N, d, bq, bkv = w.N, w.d, w.bq, w.bkv
    pairs = 0
    for b, h, i in np.ndindex(w.B, w.H, w.n_q):
        rows = min(bq, N - i * bq)
        keys = sum(min(bkv, N - int(j) * bkv) for j in kept[b, h, i])
        pairs += rows * keys
    return 4.0 * N * N * d * w.H * w.B, 4.0 * d * pairs


def test_work_counts_match_brute_force():
    # ragged last query and key blocks, the last key block kept by some rows
    w = inputs.Workload("count", 1, 3, (1, 25, 40), 64, 128, 64, "bf16", keep_count=3)
    assert w.N % w.bq and w.N % w.bkv
    rng = np.random.default_rng(0)
    kept = np.stack([np.sort(rng.choice(w.n_kv, 3, replace=False)) for _ in range(w.H * w.n_q)])
    kept = kept.reshape(1, w.H, w.n_q, 3)
    kept[0, 0, 0] = [0, 5, w.n_kv - 1]
    full, executed = bench.work_counts(w, torch.from_numpy(kept))
    want_full, want_exec = _brute(w, kept)
    assert full == want_full
    assert executed == want_exec


def test_work_counts_at_the_headline_shape():
    """Wan2.1-1.3B: 15 kept blocks everywhere, none the ragged last one."""
    w = inputs.WORKLOADS["wan13"]
    kept = torch.arange(15, dtype=torch.int32).expand(w.B, w.H, w.n_q, 15)
    full, executed = bench.work_counts(w, kept)
    assert full == 4.0 * 32760 ** 2 * 128 * 12
    assert executed == 4.0 * 128 * 12 * 32760 * 15 * 64
    assert abs(full / 6.594e12 - 1) < 1e-3


def test_reference_arm_uses_the_oracle_alone(tmp_path):
    """bench.py --impl reference: the CPU oracle on a bounded sample, its keep
    count from the oracle, and libsla.so never mapped into the process."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys, runpy; sys.argv = ['bench.py', '--impl', 'reference', '--workload', 'tiny', "
            "'--steps', '2', '--warmup', '3']; runpy.run_path('bench.py', run_name='__main__'); "
            "maps = open('/proc/self/maps').read(); print('LIBSLA_MAPPED' if 'libsla.so' in maps else 'NO_LIBSLA')")
    out = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = out.stdout.strip().splitlines()
    assert lines[-1] == "NO_LIBSLA"
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["cpu_baseline"]["kind"] == "oracle"
    assert "keep=4/16" in rec["config"]["workload"]


def test_gpus_flag_must_match_the_launcher():
    """Under a launcher, --gpus N must equal the number of ranks it started."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--impl", "reference"], cwd=root, env=env,
                         capture_output=True, text=True, timeout=120)
    assert out.returncode != 0 and "launcher started 1 ranks" in out.stderr
