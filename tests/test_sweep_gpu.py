"""Parity over the B*H*N = 131072 sweep (N in {512 ... 65536}, d in {64, 128, 256}, causal and not)
at full size, in the launch configuration the bench uses.

Every point runs the whole workload on the GPU.  Checks against the fp64 oracle, element by
element:
  * forward rows (O and L) sampled from the first and last head, computed row by row;
  * dQ of the same rows, row by row;
  * dK and dV of sampled KEY rows of the last head (column sums over every query row, with L and
    D of all rows computed in blocks), at every N;
  * for N <= 8192 also the complete dQ, dK and dV of the first head.
Sampled gradients are compared with the backward tolerance relative to the largest reference
value among the sampled rows (never larger than the whole tensor's, so the check is at least as
strict as the stated one).
"""
import numpy as np
import pytest

import attn_inputs as ai
from oracle import (attention_backward, attention_dkdv_key_rows, attention_dq_rows,
                    attention_forward, attention_row_stats, attention_rows)
from parity import assert_bwd, assert_fwd, bwd_report, BWD_REL, to_np
from gpu_util import cuda_inputs

pytestmark = pytest.mark.gpu

SPLITS = {512: (16, 16), 2048: (4, 16), 8192: (1, 16), 32768: (1, 4), 65536: (1, 2)}


def sample_rows(N, seed):
    fixed = [0, 1, 2, 63, 64, 127, 128, N // 2, N - 129, N - 128, N - 2, N - 1]
    rng = np.random.default_rng(seed)
    extra = rng.integers(0, N, size=12).tolist()
    return np.unique(np.clip(np.array(fixed + extra), 0, N - 1))


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("N", [512, 2048, 8192, 32768, 65536])
def test_sweep_point(N, d, causal):
    import torch
    import exact_io_aware_43_b200 as fa
    B, H = SPLITS[N]
    dev, f64 = cuda_inputs(B, H, N, d, seed=N + d + int(causal))
    s = ai.default_scale(d)
    o, lse = fa.forward(dev["q"], dev["k"], dev["v"], causal, s)
    dq, dk, dv = fa.backward(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], causal, s)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    what = f"N={N} d={d} causal={causal}"
    heads = [(0, 0), (B - 1, H - 1)]
    rows = sample_rows(N, N + d)
    o_h, lse_h, dq_h = {}, {}, {}
    for (b, h) in heads:
        o_h[(b, h)] = to_np(o[b, h, rows])
        lse_h[(b, h)] = to_np(lse[b, h, rows])
        dq_h[(b, h)] = to_np(dq[b, h, rows])
    for (b, h) in heads:
        qh, kh, vh, doh = (f64[t][b, h] for t in ("q", "k", "v", "do"))
        O_r, L_r = attention_rows(qh, kh, vh, rows, causal, s)
        assert_fwd(o_h[(b, h)], O_r, lse_h[(b, h)], L_r, f"{what} head {(b, h)} rows")
        dq_r = attention_dq_rows(qh, kh, vh, doh, rows, causal, s)
        e = bwd_report(dq_h[(b, h)], dq_r)
        assert e <= BWD_REL, f"{what} head {(b, h)}: dQ rows relative error {e:.3e}"
    if N <= 8192:
        sl = (slice(0, 1), slice(0, 1))
        O, L = attention_forward(f64["q"][sl], f64["k"][sl], f64["v"][sl], causal, s)
        g = attention_backward(f64["q"][sl], f64["k"][sl], f64["v"][sl], O, L, f64["do"][sl],
                               causal, s)
        assert_bwd((to_np(dq[0, 0]), to_np(dk[0, 0]), to_np(dv[0, 0])),
                   tuple(x[0, 0] for x in g), f"{what} head 0 full backward")
    b, h = heads[-1]
    keys = sample_rows(N, N + d + 1)
    dk_h, dv_h = to_np(dk[b, h, keys]), to_np(dv[b, h, keys])
    qh, kh, vh, doh = (f64[t][b, h] for t in ("q", "k", "v", "do"))
    stats = attention_row_stats(qh, kh, vh, doh, causal, s)
    dk_r, dv_r = attention_dkdv_key_rows(qh, kh, vh, doh, keys, causal, s, stats=stats)
    for name, g, r in (("dK", dk_h, dk_r), ("dV", dv_h, dv_r)):
        e = bwd_report(g, r)
        assert e <= BWD_REL, f"{what} head {(b, h)}: {name} key rows relative error {e:.3e}"
