"""fa_fwd_bwd_host (host buffers in and out, copies overlapped with the kernels by head chunks)
gives what fa_fwd and fa_bwd give on device buffers: O, L, dK, dV bit for bit (same kernels on
the same heads), dQ to fp32-atomic reordering (its reduction order may differ between runs), and
both agree with the oracle."""
import numpy as np
import pytest

import attn_inputs as ai
from oracle import attention_backward, attention_forward
from parity import assert_bwd, to_np
from gpu_util import cuda_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("chunks", [1, 3, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_host_pipeline_matches_device_path(chunks, causal):
    import torch
    import exact_io_aware_43_b200 as fa
    B, H, N, d = 2, 4, 700, 128
    dev, f64 = cuda_inputs(B, H, N, d, seed=chunks + 10 * causal)
    s = ai.default_scale(d)
    o_ref, l_ref = fa.forward(dev["q"], dev["k"], dev["v"], causal, s)
    g_ref = fa.backward(dev["q"], dev["k"], dev["v"], o_ref, l_ref, dev["do"], causal, s)
    torch.cuda.synchronize()
    host = {k: v.cpu().pin_memory() for k, v in dev.items()}
    o_h = torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory()
    l_h = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    dq, dk, dv = fa.forward_backward_host(host["q"], host["k"], host["v"], host["do"], causal, s,
                                          chunks=chunks, out=o_h, lse=l_h)
    assert fa.fa_device_status() == 0
    assert torch.equal(o_h, o_ref.cpu()) and torch.equal(l_h, l_ref.cpu())
    assert torch.equal(dk, g_ref[1].cpu()) and torch.equal(dv, g_ref[2].cpu())
    assert torch.allclose(dq.float(), g_ref[0].cpu().float(), rtol=1e-2, atol=1e-3)
    O, L = attention_forward(f64["q"], f64["k"], f64["v"], causal, s)
    R = attention_backward(f64["q"], f64["k"], f64["v"], O, L, f64["do"], causal, s)
    assert_bwd((to_np(dq), to_np(dk), to_np(dv)), R, f"host pipeline chunks={chunks}")


def test_host_pipeline_repeated_calls_reuse_buffers():
    """Back-to-back calls with one device buffer: the second call's copies wait for the first."""
    import torch
    import exact_io_aware_43_b200 as fa
    B, H, N, d = 1, 6, 512, 64
    devs = [cuda_inputs(B, H, N, d, seed=s)[0] for s in (1, 2)]
    hosts = [{k: v.cpu().pin_memory() for k, v in x.items()} for x in devs]
    buf = torch.empty(fa.fa_fwd_bwd_host_device_bytes(B, H, N, d, 3), dtype=torch.uint8,
                      device="cuda")
    outs = []
    for h in hosts:
        outs.append([t.clone() for t in fa.forward_backward_host(
            h["q"], h["k"], h["v"], h["do"], True, chunks=3, device_buffer=buf)])
    for x, got in zip(devs, outs):
        o, l = fa.forward(x["q"], x["k"], x["v"], True)
        ref = fa.backward(x["q"], x["k"], x["v"], o, l, x["do"], True)
        torch.cuda.synchronize()
        assert torch.equal(got[1], ref[1].cpu()) and torch.equal(got[2], ref[2].cpu())
