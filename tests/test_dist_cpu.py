"""The benchmark's multi-process path on CPU: two gloo ranks, as bench.py runs
one process per GPU (no GPU, no data-path collective; only the timing is
shared)."""
import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def _timing_worker(rank, world, port, values, out_q):
    dist = _init(rank, world, port, 60)
    try:
        from sparse_linear_attention_b200 import dist_timing
        r, w, _ = dist_timing.world_info()
        got = dist_timing.max_over_ranks(values[rank])
        dist_timing.barrier()
        out_q.put((rank, r, w, got, dist_timing.job_throughput(100.0, got, w), dist_timing.reports(rank),
                   dist_timing.distributed()))
    finally:
        dist.destroy_process_group()


def _leaving_worker(rank, world, port, out_q):
    dist = _init(rank, world, port, 5)
    from sparse_linear_attention_b200 import dist_timing
    if rank == 1:
        out_q.put((rank, "left"))
        out_q.close()
        out_q.join_thread()  # the message is flushed before the process goes
        os._exit(0)  # leaves between steps, before the collective
    try:
        dist_timing.max_over_ranks(1.0)
        out_q.put((rank, "returned"))
    except Exception as e:  # the collective must end with an error, not wait forever
        out_q.put((rank, type(e).__name__))


def _run(target, args_of, n=2, timeout=120):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=args_of(r, port, q)) for r in range(n)]
    for p in procs:
        p.start()
    res = [q.get(timeout=timeout) for _ in range(n)]
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    return sorted(res), [p.exitcode for p in procs]


def test_two_ranks_take_the_max_and_rank0_reports():
    values = [3.5, 7.25]
    res, codes = _run(_timing_worker, lambda r, port, q: (r, 2, port, values, q))
    assert codes == [0, 0]
    for rank, r, w, got, tput, rep, dist_on in res:
        assert (r, w, dist_on) == (rank, 2, True)
        assert got == 7.25
        assert tput == pytest.approx(100.0 * 2 / 7.25e-3)
        assert rep == (rank == 0)


def test_a_rank_that_leaves_ends_the_others_collective_with_an_error():
    res, _ = _run(_leaving_worker, lambda r, port, q: (r, 2, port, q))
    assert res[1] == (1, "left")
    assert res[0][0] == 0 and res[0][1] != "returned", res


def test_single_process_needs_no_group():
    from sparse_linear_attention_b200 import dist_timing
    assert not dist_timing.distributed()
    assert dist_timing.max_over_ranks(2.5) == 2.5
    assert dist_timing.job_throughput(10.0, 2.0, 1) == pytest.approx(5000.0)
    with pytest.raises(ValueError):
        dist_timing.job_throughput(1.0, 0.0, 1)


_RANK_SCRIPT = '''
import datetime, json, os, sys
sys.path.insert(0, {root!r})
from sparse_linear_attention_b200 import dist_timing
n = int(sys.argv[sys.argv.index("--gpus") + 1])
if n > 1 and not dist_timing.launched():
    raise SystemExit(dist_timing.run_ranks(os.path.abspath(__file__), sys.argv[1:], n, timeout_s=120))
import torch.distributed as dist
rank, world, _ = dist_timing.world_info()
assert world == n
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=30))
got = dist_timing.max_over_ranks(float(rank + 1))
dist.destroy_process_group()
if dist_timing.reports(rank):
    print(json.dumps({{"n_gpus": world, "max": got}}), flush=True)
'''


def test_gpus_flag_starts_its_own_ranks(tmp_path):
    """bench.py's launcher path: `--gpus 2` outside torchrun starts two ranks of
    the same script under torchrun (gloo here), every rank sees world size 2,
    and rank 0 alone reports the max over ranks."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    script = tmp_path / "ranks.py"
    script.write_text(_RANK_SCRIPT.format(root=root))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, str(script), "--gpus", "2"], capture_output=True, text=True,
                         timeout=180, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    recs = [json.loads(x) for x in out.stdout.splitlines() if x.startswith("{")]
    assert recs == [{"n_gpus": 2, "max": 2.0}]


def test_launcher_command_uses_loopback_rendezvous():
    from sparse_linear_attention_b200 import dist_timing
    cmd = dist_timing.launcher_argv("bench.py", ["--gpus", "4"], 4, 29511)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd and "--master-port=29511" in cmd
    assert cmd[-3:] == ["bench.py", "--gpus", "4"]
