"""Grouped-query attention (GQA / MQA) parity: fa_fwd_gqa and fa_bwd_gqa (CUDA, through the C ABI)
against the fp64 grouped oracle, with the same tolerances as the one-head-per-key/value tests.

Cases span d = 64 / 128 / 256, causal and not, ragged N, group sizes 1 (through the grouped entry
point), 2, 3, 4 and 8, and multi-query attention (one key/value head).  A larger causal d = 128 case
checks one whole group (its key/value head's dK and dV need every query head of the group)."""
import ctypes

import numpy as np
import pytest

import attn_inputs as ai
from oracle import attention_backward_gqa, attention_forward_gqa
from parity import assert_bwd, assert_fwd, to_np
from gpu_util import cuda_inputs

pytestmark = pytest.mark.gpu


def run_gpu(B, H, Hkv, N, d, causal, seed=0, sigma_qk=1.0):
    import torch
    import exact_io_aware_43_b200 as fa
    dev, f64 = cuda_inputs(B, H, N, d, seed, sigma_qk, kv_heads=Hkv)
    s = ai.default_scale(d)
    o, lse = fa.forward(dev["q"], dev["k"], dev["v"], causal, s)
    dq, dk, dv = fa.backward(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], causal, s)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    return (to_np(o), to_np(lse)), (to_np(dq), to_np(dk), to_np(dv)), f64, s


def check(B, H, Hkv, N, d, causal, seed=0, sigma_qk=1.0):
    (o, lse), g, f64, s = run_gpu(B, H, Hkv, N, d, causal, seed, sigma_qk)
    O, L = attention_forward_gqa(f64["q"], f64["k"], f64["v"], causal, s)
    what = f"B={B} H={H} H_kv={Hkv} N={N} d={d} causal={causal}"
    assert_fwd(o, O, lse, L, what)
    R = attention_backward_gqa(f64["q"], f64["k"], f64["v"], O, L, f64["do"], causal, s)
    assert_bwd(g, R, what)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H,Hkv,N", [(4, 2, 300), (6, 3, 129), (8, 1, 200), (4, 4, 64),
                                     (8, 2, 1)])
def test_gqa_parity(H, Hkv, N, d, causal):
    check(2 if N < 256 else 1, H, Hkv, N, d, causal, seed=H * 10 + Hkv + N)


def test_gqa_peaky_softmax():
    check(1, 8, 2, 512, 128, False, seed=5, sigma_qk=3.0)


def test_gqa_group_of_eight_long_causal():
    """H = 16 query heads on 2 key/value heads, N = 2048, d = 128 causal: key/value head 0 and the
    8 query heads that read it, checked completely (the oracle runs on that group only)."""
    (o, lse), (dq, dk, dv), f64, s = run_gpu(1, 16, 2, 2048, 128, True, seed=9)
    G = 8
    q, k, v, do = (f64[n][:, :G] if n in ("q", "do") else f64[n][:, :1]
                   for n in ("q", "k", "v", "do"))
    O, L = attention_forward_gqa(q, k, v, True, s)
    assert_fwd(o[:, :G], O, lse[:, :G], L, "group 0 forward")
    R = attention_backward_gqa(q, k, v, O, L, do, True, s)
    assert_bwd((dq[:, :G], dk[:, :1], dv[:, :1]), R, "group 0 backward")


def test_grouped_entry_with_one_head_per_group_matches_plain_entry():
    """fa_fwd_gqa / fa_bwd_gqa with H_kv = H run the same kernels as fa_fwd / fa_bwd: bit-equal."""
    import torch
    import exact_io_aware_43_b200 as fa
    B, H, N, d = 1, 4, 384, 128
    dev, _ = cuda_inputs(B, H, N, d, seed=21)
    s = ai.default_scale(d)
    st = torch.cuda.current_stream().cuda_stream
    outs = []
    for grouped in (False, True):
        o = torch.empty_like(dev["q"])
        lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
        args = (dev["q"].data_ptr(), dev["k"].data_ptr(), dev["v"].data_ptr(), o.data_ptr(),
                lse.data_ptr())
        rc = (fa.fa_fwd_gqa(*args, B, H, H, N, d, True, s, st) if grouped else
              fa.fa_fwd(*args, B, H, N, d, True, s, st))
        assert rc == 0
        ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
        g = [torch.empty_like(dev["q"]) for _ in range(3)]
        bargs = args + (dev["do"].data_ptr(), g[0].data_ptr(), g[1].data_ptr(), g[2].data_ptr())
        rc = (fa.fa_bwd_gqa(*bargs, B, H, H, N, d, True, s, ws.data_ptr(), ws.numel(), st)
              if grouped else
              fa.fa_bwd(*bargs, B, H, N, d, True, s, ws.data_ptr(), ws.numel(), st))
        assert rc == 0
        torch.cuda.synchronize()
        outs.append([o, lse] + g)
    for a, b in zip(*outs):
        assert torch.equal(a, b)
