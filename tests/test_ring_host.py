"""Ring (context-parallel) attention, host logic on CPU: the schedule, and the whole ring run by
two and three gloo ranks with the partial and merge steps taken from the fp64 oracle, against
the oracle's attention over the full sequence.  (The CUDA partial and merge steps are checked
on the GPU in test_ring_gpu.py.)"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from exact_io_aware_43_b200.ring import ring_steps

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_schedule_causal_and_full():
    for W in (1, 2, 3, 5):
        for r in range(W):
            full = ring_steps(r, W, False)
            assert sorted(j for _, j, _ in full) == list(range(W))
            assert all(m == "full" for _, _, m in full)
            causal = ring_steps(r, W, True)
            assert [j for _, j, _ in causal] == [j for _, j, _ in full]  # same transfers
            seen = {j: m for _, j, m in causal}
            assert seen[r] == "causal"
            assert all(seen[j] == "full" for j in range(r))
            assert all(seen[j] == "skip" for j in range(r + 1, W))
            # step s holds the shard of rank r - s: each shard moves one rank on per step
            assert [j for _, j, _ in causal] == [(r - s) % W for s in range(W)]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _oracle_partial(q, k, v, causal, scale):
    from oracle import attention_forward_rect
    O, L = attention_forward_rect(q.numpy(), k.numpy(), v.numpy(), causal, scale)
    return O, L


def _lse_merge(parts):
    L = np.logaddexp.reduce(np.stack([p[1] for p in parts]), axis=0)
    O = sum(np.exp(p[1] - L)[..., None] * p[0] for p in parts)
    return O, L


def _worker(rank, world, port, causal, q_out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from exact_io_aware_43_b200.ring import ring_forward
    from oracle import attention_forward
    rng = np.random.default_rng(5)
    n, B, H, Hkv, d = 7, 1, 4, 2, 8
    N = world * n
    q = rng.standard_normal((B, H, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    sl = slice(rank * n, (rank + 1) * n)
    O, L = ring_forward(torch.from_numpy(q[:, :, sl].copy()), torch.from_numpy(k[:, :, sl].copy()),
                        torch.from_numpy(v[:, :, sl].copy()), causal, 0.4, _oracle_partial,
                        _lse_merge)
    G = H // Hkv
    Of, Lf = attention_forward(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1), causal, 0.4)
    q_out.put((rank, float(np.abs(O - Of[:, :, sl]).max()), float(np.abs(L - Lf[:, :, sl]).max())))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_over_gloo_ranks_equals_full_attention(world, causal):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, eo, el in out:
        assert eo <= 1e-12 and el <= 1e-12, (rank, eo, el)
