"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory (for example a
program whose pooled allocator already owns almost all of the GPU, or a host that forbids
allocation during a step).  Its workspace is the library's static 32 MiB device array.

The GPU test calls the entry point through the C ABI twice in a row.  Each result is compared
with the fp64 oracle within the backward tolerance the other tests use, and with fa_bwd given a
caller-provided workspace: dK and dV bit for bit (the same kernels run, and they are
deterministic when every query head has its own key/value head), dQ within the tolerance (its
fp32 reduction order varies).  The second call checks that scratch left over from the first call
does not leak into the result.  This file is collected last so a stop-at-first-failure run has
already run every other test.
"""
import numpy as np
import pytest

import exact_io_aware_43_b200 as fa
from oracle import attention_backward, attention_forward
from parity import BWD_REL, assert_bwd, bwd_report, to_np
from gpu_util import cuda_inputs


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,d,causal", [(2, 4, 777, 128, True), (3, 2, 500, 64, False),
                                             (1, 2, 300, 256, True)])
def test_noalloc_matches_fa_bwd_twice(B, H, N, d, causal):
    import torch
    assert fa.fa_bwd_workspace_size(B, H, N, d) <= fa.FA_NOALLOC_SCRATCH_BYTES
    dev, f64 = cuda_inputs(B, H, N, d, seed=21)
    q, k, v, do = dev["q"], dev["k"], dev["v"], dev["do"]
    s = float(np.float32(1.0 / np.sqrt(d)))
    o, lse = fa.forward(q, k, v, causal, s)
    ref_dq, ref_dk, ref_dv = fa.backward(q, k, v, o, lse, do, causal, s)
    torch.cuda.synchronize()
    O, L = attention_forward(f64["q"], f64["k"], f64["v"], causal, s)
    exact = attention_backward(f64["q"], f64["k"], f64["v"], O, L, f64["do"], causal, s)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        rc = fa.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                               lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                               dv.data_ptr(), B, H, N, d, causal, s, stream)
        assert rc == fa.FA_OK, fa.fa_last_error()
        torch.cuda.synchronize()
        assert fa.fa_device_status() == fa.FA_OK
        assert_bwd(tuple(to_np(t) for t in (dq, dk, dv)), exact, f"fa_bwd_noalloc call {call}")
        assert torch.equal(dk, ref_dk), f"call {call}: dk differs from fa_bwd's"
        assert torch.equal(dv, ref_dv), f"call {call}: dv differs from fa_bwd's"
        err = bwd_report(to_np(dq), to_np(ref_dq))
        assert err <= BWD_REL, f"call {call}: dq differs from fa_bwd's by {err:.3e}"


def test_noalloc_rejects_shapes_beyond_the_scratch():
    """The long-context shape needs ~145 MB of workspace: rejected on the host, nothing launched."""
    A = 1 << 20
    need = fa.fa_bwd_workspace_size(2, 16, 8192, 128)
    assert need > fa.FA_NOALLOC_SCRATCH_BYTES
    rc = fa.fa_bwd_noalloc(A, A, A, A, A, A, A, A, A, 2, 16, 8192, 128, 1, 0.088, None)
    assert rc == fa.FA_ERR_WORKSPACE
    assert "static" in fa.fa_last_error()
