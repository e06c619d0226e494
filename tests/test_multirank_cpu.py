"""The multi-process (one process per GPU) path of bench.py, on CPU with gloo ranks.

Every rank runs its own replica of the workload on its own seeded batch; the only
collectives are the barrier around the timed region and the max over ranks of the
device time. These tests run that host logic with world_size 2 on the gloo backend.
"""
import hashlib
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from sparse_windowed_atom_b200 import workloads
    r = bench.Ranks("gloo", timeout_s=60)
    r.barrier()
    slowest = r.max(float(rank * 10 + 3))
    rate = r.job_rate(100.0, 2.0)           # 100 units per rank per 2 ms step
    spec = workloads.tiny_spec("af3", "encoder", B=1, A=40, T=8, K=10, C=16, S=8, H=2, D=8,
                               P=4, M=16, U=12)
    w = workloads.make_inputs(spec, seed=r.seed())
    digest = hashlib.sha256(w["activations"]["atom"].tobytes()).hexdigest()
    r.barrier()
    q.put((rank, slowest, rate, digest))
    r.close()


def test_two_gloo_ranks_time_as_max_and_count_all_units():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [13.0, 13.0]                 # max over ranks, on every rank
    assert all(abs(r[2] - 100.0 * world / 2e-3) < 1e-6 for r in res)
    assert res[0][3] != res[1][3]                             # each rank draws its own batch


def test_reference_arm_runs_on_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                         text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == ""
