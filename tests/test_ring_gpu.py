"""Ring (context-parallel) attention on one GPU: every rank of a W-rank ring is played in turn
(no transfers; the schedule is ring_steps), computing its partials over each key shard with
fa_fwd_partial and merging them with fa_merge_partials, against the fp64 oracle's attention over
the full sequence.  The transfers themselves are covered on CPU (test_ring_host.py)."""
import numpy as np
import pytest

import attn_inputs as ai
from oracle import attention_forward_gqa
from parity import assert_fwd, to_np
from gpu_util import cuda_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("W,n,d,Hkv", [(2, 300, 128, 4), (3, 256, 64, 2), (4, 129, 256, 4),
                                       (2, 1024, 128, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_ranks_on_one_gpu(W, n, d, Hkv, causal):
    import torch
    import exact_io_aware_43_b200 as fa
    from exact_io_aware_43_b200.ring import cuda_merge, cuda_partial, ring_steps
    B, H = 1, 4
    N = W * n
    dev, f64 = cuda_inputs(B, H, N, d, seed=W + n, with_do=False, kv_heads=Hkv)
    s = ai.default_scale(d)
    O, L = attention_forward_gqa(f64["q"], f64["k"], f64["v"], causal, s)
    for r in range(W):
        qs = dev["q"][:, :, r * n:(r + 1) * n].contiguous()
        parts = []
        for (_, j, mode) in ring_steps(r, W, causal):
            if mode == "skip":
                continue
            ks = dev["k"][:, :, j * n:(j + 1) * n].contiguous()
            vs = dev["v"][:, :, j * n:(j + 1) * n].contiguous()
            parts.append(cuda_partial(qs, ks, vs, mode == "causal", s))
        o, lse = cuda_merge(parts)
        torch.cuda.synchronize()
        assert fa.fa_device_status() == 0
        sl = slice(r * n, (r + 1) * n)
        assert_fwd(to_np(o), O[:, :, sl], to_np(lse), L[:, :, sl], f"ring rank {r} of {W}")


def test_partial_with_no_weight_changes_nothing():
    """A partial whose logsumexp is -inf (a key shard the rows cannot see) has weight 0 in the
    merge: merging it beside a real partial of 128 queries over 256 keys changes no bit."""
    import torch
    from exact_io_aware_43_b200.ring import cuda_merge, cuda_partial
    dev, _ = cuda_inputs(1, 2, 256, 128, seed=9, with_do=False)
    q, k, v = dev["q"][:, :, :128].contiguous(), dev["k"], dev["v"]
    a = cuda_partial(q, k, v, False, 0.1)
    o1, l1 = cuda_merge([a])
    o2, l2 = cuda_merge([a, (torch.zeros_like(a[0]), torch.full_like(a[1], float("-inf")))])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
