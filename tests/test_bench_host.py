"""Host-side logic of the multi-GPU bench on CPU: two gloo ranks, each with its own batch seed,
agree on the slowest rank's time through the max-reduction."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    t = bench.reduce_max(1.5 + rank)
    bench.barrier()
    q.put((rank, bench.rank_seed(rank), t, bench.dist_env()))
    dist.destroy_process_group()


def test_two_rank_reduce_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    assert [o[2] for o in out] == [2.5, 2.5]          # both ranks see the max
    assert out[0][1] != out[1][1]                    # distinct batches per rank
    assert [o[3][:2] for o in out] == [(0, 2), (1, 2)]


def test_flop_count_matches_metric_definition():
    sys.path.insert(0, ROOT)
    import bench
    ff, fb = bench.flops(2, 16, 8192, 128, True)
    assert ff == 4 * 2 * 16 * 8192 ** 2 * 128 / 2
    assert fb == 2.5 * ff
    assert bench.flops(1, 1, 10, 64, False)[0] == 4 * 100 * 64


def test_reference_arm_under_two_ranks():
    """`bench.py --impl reference` under torchrun: rank 0 times the oracle and prints one JSON
    line with impl == "reference"; the other rank exits 0 without work."""
    import json
    import subprocess
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}",
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
