"""Forward parity: fa_fwd (CUDA, through the C ABI) against the fp64 oracle, element by element."""
import numpy as np
import pytest

import attn_inputs as ai
from oracle import attention_forward
from parity import assert_fwd, to_np
from gpu_util import cuda_inputs

pytestmark = pytest.mark.gpu


def run_fwd(B, H, N, d, causal, seed=0, sigma_qk=1.0, heads=None):
    import torch
    import exact_io_aware_43_b200 as fa
    dev, f64 = cuda_inputs(B, H, N, d, seed, sigma_qk, with_do=False)
    s = ai.default_scale(d)
    o, lse = fa.forward(dev["q"], dev["k"], dev["v"], causal, s)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    o, lse = to_np(o), to_np(lse)
    if heads is None:
        O_ref, L_ref = attention_forward(f64["q"], f64["k"], f64["v"], causal, s)
        return o, lse, O_ref, L_ref
    outs = []
    for (b, h) in heads:
        O_ref, L_ref = attention_forward(f64["q"][b:b + 1, h:h + 1], f64["k"][b:b + 1, h:h + 1],
                                         f64["v"][b:b + 1, h:h + 1], causal, s)
        outs.append((o[b, h], lse[b, h], O_ref[0, 0], L_ref[0, 0]))
    return outs


def test_tiny_workload_noncausal():
    o, lse, O, L = run_fwd(1, 2, 128, 64, False)
    assert_fwd(o, O, lse, L, "B=1 H=2 N=128 d=64")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 3, 64, 127, 128, 129, 200, 255, 256, 257, 383, 512, 700])
def test_ragged_lengths(N, d, causal):
    o, lse, O, L = run_fwd(1, 2, N, d, causal, seed=N)
    assert_fwd(o, O, lse, L, f"N={N} d={d} causal={causal}")


@pytest.mark.parametrize("d", [64, 128, 256])
def test_causal_row0_is_v0(d):
    """Causal row 0 sees only key 0: P~ = 1, l = 1, so O_0 = V_0 bit for bit."""
    import torch
    import exact_io_aware_43_b200 as fa
    dev, _ = cuda_inputs(2, 3, 300, d, seed=5, with_do=False)
    o, _ = fa.forward(dev["q"], dev["k"], dev["v"], True)
    torch.cuda.synchronize()
    assert torch.equal(o[:, :, 0], dev["v"][:, :, 0])


@pytest.mark.parametrize("seed", [0, 1, 2, 3, 4])
def test_gpt2_small_causal(seed):
    o, lse, O, L = run_fwd(8, 12, 1024, 64, True, seed=seed)
    assert_fwd(o, O, lse, L, f"GPT-2-small causal seed {seed}")


@pytest.mark.parametrize("sigma", [1.0, 3.0])
def test_bert_large(sigma):
    o, lse, O, L = run_fwd(16, 16, 512, 64, False, sigma_qk=sigma)
    assert_fwd(o, O, lse, L, f"BERT-large sigma_qk={sigma}")


@pytest.mark.parametrize("seed", [0, 1, 2, 3, 4])
def test_long_context_sampled_heads(seed):
    """B=2 H=16 N=8192 d=128 causal: complete check of the first and last heads; seed 0 for
    parity and seeds 1-4 as repeats."""
    for (o, lse, O, L) in run_fwd(2, 16, 8192, 128, True, seed=seed, heads=[(0, 0), (1, 15)]):
        assert_fwd(o, O, lse, L, f"long context causal seed {seed}")


def test_deterministic():
    import torch
    import exact_io_aware_43_b200 as fa
    dev, _ = cuda_inputs(2, 4, 1000, 128, seed=3, with_do=False)
    o1, l1 = fa.forward(dev["q"], dev["k"], dev["v"], True)
    o2, l2 = fa.forward(dev["q"], dev["k"], dev["v"], True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("d", [64, 128])
def test_split_tail_noncausal(d):
    """B=7 H=8 N=700 non-causal: 168 units of two query tiles on 148 SMs; the 20 units of the
    short last round run as 40 one-tile items, the last query block (rows 512..699) among them,
    its second tile ragged."""
    o, lse, O, L = run_fwd(7, 8, 700, d, False, seed=11)
    assert_fwd(o, O, lse, L, f"split tail d={d}")
