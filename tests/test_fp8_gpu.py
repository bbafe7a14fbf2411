"""FP8 (e4m3) forward parity: fa_fwd_fp8 (CUDA, through the C ABI) against the fp64 oracle on the
dequantised inputs, with the FP8 tolerance reading of tests/parity.py (every element within the
worst-case effect of rounding the softmax weights to e4m3, the mean squared error within the
rounding model's variance, and |dL| <= 1e-3)."""
import numpy as np
import pytest

import attn_inputs as ai
from oracle import attention_forward
from parity import assert_fwd_fp8, fp8_error_bounds, to_np

pytestmark = pytest.mark.gpu


def run_fp8(B, H, N, d, causal, seed=0, sigma_qk=1.0, heads=None):
    import torch
    import exact_io_aware_43_b200 as fa
    x = ai.make_inputs_fp8(B, H, N, d, seed=seed, sigma_qk=sigma_qk)
    dev = {t: torch.from_numpy(c).cuda() for t, (c, _) in x.items()}
    sc = {t: s for t, (_, s) in x.items()}
    s = ai.default_scale(d)
    o, lse = fa.forward_fp8(dev["q"], dev["k"], dev["v"], sc["q"], sc["k"], sc["v"], causal, s)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    o, lse = to_np(o), to_np(lse)
    deq = {t: sc[t] * ai.e4m3_bits_to_f64(c) for t, (c, _) in x.items()}
    out = []
    for (b, h) in (heads or [(b, h) for b in range(B) for h in range(H)]):
        qh, kh, vh = (deq[t][b, h] for t in ("q", "k", "v"))
        O, L = attention_forward(qh[None, None], kh[None, None], vh[None, None], causal, s)
        bound, var = fp8_error_bounds(qh, kh, vh, causal, s)
        out.append((o[b, h], lse[b, h], O[0, 0], L[0, 0], bound, var))
    return out


def check(res, what):
    for i, (o, lse, O, L, bound, var) in enumerate(res):
        assert_fwd_fp8(o, O, lse, L, bound, var, f"{what} head {i}")


def test_tiny_workload_noncausal():
    check(run_fp8(1, 2, 128, 64, False), "fp8 B=1 H=2 N=128 d=64")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 3, 100, 128, 129, 300, 700])
def test_ragged_lengths(N, d, causal):
    check(run_fp8(1, 2, N, d, causal, seed=N + 1), f"fp8 N={N} d={d} causal={causal}")


def test_gpt2_small_causal():
    check(run_fp8(8, 12, 1024, 64, True, heads=[(0, 0), (3, 5), (7, 11)]), "fp8 GPT-2-small")


@pytest.mark.parametrize("sigma", [1.0, 3.0])
def test_bert_large(sigma):
    check(run_fp8(16, 16, 512, 64, False, sigma_qk=sigma, heads=[(0, 0), (9, 4), (15, 15)]),
          f"fp8 BERT-large sigma_qk={sigma}")


def test_long_context_sampled_heads():
    check(run_fp8(2, 16, 8192, 128, True, heads=[(0, 0), (1, 15)]), "fp8 long context causal")


def test_causal_row0_is_v0():
    """Causal row 0 sees only key 0: its weight is exactly 2^8 before the division, so
    O_0 = bf16(v_scale * V8_0) bit for bit."""
    import torch
    import exact_io_aware_43_b200 as fa
    x = ai.make_inputs_fp8(2, 3, 300, 128, seed=5)
    dev = {t: torch.from_numpy(c).cuda() for t, (c, _) in x.items()}
    sc = {t: s for t, (_, s) in x.items()}
    o, _ = fa.forward_fp8(dev["q"], dev["k"], dev["v"], sc["q"], sc["k"], sc["v"], True)
    torch.cuda.synchronize()
    v0 = torch.from_numpy(sc["v"] * ai.e4m3_bits_to_f64(x["v"][0][:, :, 0])).to(torch.bfloat16)
    assert torch.equal(o[:, :, 0].cpu(), v0)


def test_deterministic():
    import torch
    import exact_io_aware_43_b200 as fa
    x = ai.make_inputs_fp8(2, 4, 1000, 128, seed=3)
    dev = {t: torch.from_numpy(c).cuda() for t, (c, _) in x.items()}
    sc = [s for _, s in x.values()]
    o1, l1 = fa.forward_fp8(dev["q"], dev["k"], dev["v"], *sc, True)
    o2, l2 = fa.forward_fp8(dev["q"], dev["k"], dev["v"], *sc, True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fma_pipe_exp2_within_its_bound():
    """The FP8 softmax's FMA-pipe exponential (fa_selftest_exp2_fma runs the device function)
    against exp2 in fp64: relative error at most 7.5e-5 (the fitted cubic's bound on [-1/2, 1/2],
    plus float32 rounding of the reduction and the result) wherever the result is a normal float.
    Inputs at or below -126 clamp there; the cubic's value just under 1 then lands in the
    subnormal range, where inserting the exponent drops the implicit bit, so the result is only
    within 2e-4 of 2^-126 -- a positive value of order 1e-38 that the e4m3 rounding of the
    weights (to 0) and the fp32 row sum both absorb."""
    import torch
    import exact_io_aware_43_b200 as fa
    x = np.concatenate([np.linspace(-125.0, 20.0, 1 << 20), np.array([0.0, 8.0, -1.0, 0.5, -0.5]),
                        np.random.default_rng(0).uniform(-30.0, 8.5, 1 << 18)]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    y = torch.empty_like(xd)
    assert fa.fa_selftest_exp2_fma(xd.data_ptr(), y.data_ptr(), x.size,
                                   torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    torch.cuda.synchronize()
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y.cpu().numpy().astype(np.float64) / ref - 1.0)
    assert rel.max() <= 7.5e-5 + 2.4e-7, rel.max()
    low = torch.tensor([-126.0, -200.0, -1e30], device="cuda")
    out = torch.empty_like(low)
    assert fa.fa_selftest_exp2_fma(low.data_ptr(), out.data_ptr(), 3, None) == fa.FA_OK
    torch.cuda.synchronize()
    assert np.allclose(out.cpu().numpy(), 2.0 ** -126, rtol=2e-4, atol=0)
