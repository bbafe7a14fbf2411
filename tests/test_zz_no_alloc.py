"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory (for example a
program whose pooled allocator already owns almost all of the GPU, or a host that forbids
allocation during a step).  Its workspace is the library's static 32 MiB device array.

The GPU test calls the entry point through the C ABI twice in a row and compares each result with
fa_bwd given a caller-provided workspace, within the backward tolerance the other tests use.
The second call checks that scratch left over from the first call does not leak into the result.
This file is collected last so a stop-at-first-failure run has already run every other test.
"""
import numpy as np
import pytest

import exact_io_aware_43_b200 as fa
from parity import BWD_REL, bwd_report, to_np
from gpu_util import cuda_inputs


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,d,causal", [(2, 4, 777, 128, True), (3, 2, 500, 64, False),
                                             (1, 2, 300, 256, True)])
def test_noalloc_matches_fa_bwd_twice(B, H, N, d, causal):
    import torch
    assert fa.fa_bwd_workspace_size(B, H, N, d) <= fa.FA_NOALLOC_SCRATCH_BYTES
    dev, _ = cuda_inputs(B, H, N, d, seed=21)
    q, k, v, do = dev["q"], dev["k"], dev["v"], dev["do"]
    o, lse = fa.forward(q, k, v, causal)
    ref = fa.backward(q, k, v, o, lse, do, causal)
    torch.cuda.synchronize()
    ref = [to_np(t) for t in ref]
    s = float(np.float32(1.0 / np.sqrt(d)))
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        rc = fa.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                               lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                               dv.data_ptr(), B, H, N, d, causal, s, stream)
        assert rc == fa.FA_OK, fa.fa_last_error()
        torch.cuda.synchronize()
        assert fa.fa_device_status() == fa.FA_OK
        for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            err = bwd_report(to_np(g), r)
            assert err <= BWD_REL, f"call {call}: {name} differs from fa_bwd by {err:.3e}"


def test_noalloc_rejects_shapes_beyond_the_scratch():
    """The long-context shape needs ~130 MB of workspace: rejected on the host, nothing launched."""
    A = 1 << 20
    need = fa.fa_bwd_workspace_size(2, 16, 8192, 128)
    assert need > fa.FA_NOALLOC_SCRATCH_BYTES
    rc = fa.fa_bwd_noalloc(A, A, A, A, A, A, A, A, A, 2, 16, 8192, 128, 1, 0.088, None)
    assert rc == fa.FA_ERR_WORKSPACE
    assert "static" in fa.fa_last_error()
