"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The attention path shards into independent replicas (no data-path
collective): each rank draws its own seeded problem, the job time is the max
over ranks, and the job throughput counts every rank's flops.  The reference
arm runs on rank 0 only.
"""
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        import bench
        from tiled_attention_16_b200.workloads import WORKLOADS, make_inputs
        wl = bench.rank_workload(WORKLOADS["tiny"], rank)
        x = make_inputs(wl)[0]
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        mx = bench.max_over_ranks(ms, ws, torch.device("cpu"))
        val = bench.job_tflops(wl.flops_fwd() + wl.flops_bwd(), ws, mx)
        q.put((rank, wl.seed, float(x.float().sum()), mx, val))
    finally:
        dist.destroy_process_group()


def test_replicas_max_over_ranks_gloo():
    ws = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(ws))
    (r0, s0, x0, m0, v0), (r1, s1, x1, m1, v1) = res
    assert (r0, r1) == (0, 1)
    assert s1 == s0 + 1 and x0 != x1          # independent problems
    assert m0 == m1 == 15.0                    # max over ranks
    assert v0 == v1
    import bench
    from tiled_attention_16_b200.workloads import WORKLOADS
    wl = WORKLOADS["tiny"]
    assert abs(v0 - 2 * (wl.flops_fwd() + wl.flops_bwd()) / 15e-3 / 1e12) < 1e-9


def test_reference_arm_non_zero_rank_exits_clean():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
