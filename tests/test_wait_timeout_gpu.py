"""Failure detection on the GPU without a fault: a bounded wait that runs out.

``libfattn_starve.so`` is the library built with one change (FA_TEST_STARVE) and a 1 ms wait
bound: in the forward, CTA 0's producer warp never issues the second K/V tile of its first unit;
in the d = 256 backward (CTA pairs), CTA 1 of the first cluster never issues its second dO tile.
Nothing is left in flight -- the copies it did issue are drained before the CTA exits -- so the
MMA warp's bounded wait for that tile simply runs out.  The kernel must then record
FA_ERR_TIMEOUT in its device status word, let every role of the CTA fall through to the teardown
(tensor memory released, issued copies and MMAs drained) and return, leaving the GPU context
usable: a normal call right after it must still meet the parity bound against the oracle.
"""
import ctypes
import os
import re
import time

import pytest

import attn_inputs as ai
import exact_io_aware_43_b200 as fa
from exact_io_aware_43_b200.build import STARVE_PATH
from oracle import attention_backward, attention_forward
from parity import assert_bwd, assert_fwd, to_np
from gpu_util import cuda_inputs

pytestmark = pytest.mark.gpu


def starve_lib():
    if not os.path.exists(STARVE_PATH):
        pytest.fail(f"{STARVE_PATH} is missing; build with `python -m exact_io_aware_43_b200.build`")
    L = ctypes.CDLL(STARVE_PATH)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
    L.fa_fwd.restype = i
    L.fa_device_status.argtypes = [vp]
    L.fa_device_status.restype = i
    L.fa_last_error.argtypes = []
    L.fa_last_error.restype = ctypes.c_char_p
    sz = ctypes.c_size_t
    L.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    L.fa_bwd_workspace_size.restype = sz
    L.fa_bwd.argtypes = [vp] * 9 + [i] * 5 + [f, vp, sz, vp]
    L.fa_bwd.restype = i
    return L


def test_starved_wait_reports_timeout_and_context_survives():
    import torch
    L = starve_lib()
    # one head, N = 1024, d = 128, no mask: 4 units of 256 queries x 8 key tiles; CTA 0's first
    # unit needs its second key tile, which never comes
    B, H, N, d = 1, 1, 1024, 128
    dev, _ = cuda_inputs(B, H, N, d, seed=40, with_do=False)
    o = torch.empty_like(dev["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    rc = L.fa_fwd(dev["q"].data_ptr(), dev["k"].data_ptr(), dev["v"].data_ptr(), o.data_ptr(),
                  lse.data_ptr(), B, H, N, d, 0, ai.default_scale(d), stream)
    assert rc == fa.FA_OK, L.fa_last_error()
    status = L.fa_device_status(stream)  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert status == fa.FA_ERR_TIMEOUT, (status, L.fa_last_error())
    # whichever role noticed first: the MMA warp waiting for K of the second tile (site 16) or a
    # softmax warpgroup waiting for the second score tile (site 20)
    msg = L.fa_last_error().decode()
    assert ("site 16" in msg) or ("site 20" in msg), msg
    # the wait gave up after about 1 ms and the teardown did not wait out its own bound
    assert elapsed < 1.0, elapsed
    # the status word was read and cleared: a second read reports nothing new
    assert L.fa_device_status(stream) == fa.FA_OK

    # the context is intact: the product library runs a forward + backward that meets parity
    dev, f64 = cuda_inputs(1, 2, 300, 128, seed=41)
    s = ai.default_scale(128)
    o, lse = fa.forward(dev["q"], dev["k"], dev["v"], True, s)
    dq, dk, dv = fa.backward(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], True, s)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    O, Lr = attention_forward(f64["q"], f64["k"], f64["v"], True, s)
    assert_fwd(to_np(o), O, to_np(lse), Lr, "after the starved call")
    g = attention_backward(f64["q"], f64["k"], f64["v"], O, Lr, f64["do"], True, s)
    assert_bwd(tuple(to_np(t) for t in (dq, dk, dv)), g, "after the starved call")


def test_starve_build_is_otherwise_the_same_library():
    """A problem that never reaches the starved tile (one key tile per unit) runs normally in the
    test build, so the only difference is the one left-out load."""
    import torch
    L = starve_lib()
    B, H, N, d = 1, 2, 100, 128
    dev, f64 = cuda_inputs(B, H, N, d, seed=42, with_do=False)
    o = torch.empty_like(dev["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    s = ai.default_scale(d)
    rc = L.fa_fwd(dev["q"].data_ptr(), dev["k"].data_ptr(), dev["v"].data_ptr(), o.data_ptr(),
                  lse.data_ptr(), B, H, N, d, 1, s, stream)
    assert rc == fa.FA_OK, L.fa_last_error()
    assert L.fa_device_status(stream) == fa.FA_OK
    O, Lr = attention_forward(f64["q"], f64["k"], f64["v"], True, s)
    assert_fwd(to_np(o), O, to_np(lse), Lr, "starve build, single key tile")


def test_starved_pair_backward_reports_timeout_and_context_survives():
    """The d = 256 backward runs on two-CTA clusters that exchange tiles through each other's
    shared memory.  With one dO tile of the first cluster never issued, a bounded wait runs out
    on one CTA, the abort reaches the other through its abort flag, both tear down (each sender
    waits, bounded, for the hand-back of the tiles it sent, then the cluster barrier), and the
    call returns with FA_ERR_TIMEOUT and a usable context."""
    import torch
    L = starve_lib()
    B, H, N, d = 1, 1, 256, 256
    dev, f64 = cuda_inputs(B, H, N, d, seed=43)
    s = ai.default_scale(d)
    o, lse = fa.forward(dev["q"], dev["k"], dev["v"], True, s)  # product library: O and L
    torch.cuda.synchronize()
    dq, dk, dv = (torch.empty_like(dev[t]) for t in ("q", "k", "v"))
    ws = torch.empty(L.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    rc = L.fa_bwd(dev["q"].data_ptr(), dev["k"].data_ptr(), dev["v"].data_ptr(), o.data_ptr(),
                  lse.data_ptr(), dev["do"].data_ptr(), dq.data_ptr(), dk.data_ptr(),
                  dv.data_ptr(), B, H, N, d, 1, s, ws.data_ptr(), ws.numel(), stream)
    assert rc == fa.FA_OK, L.fa_last_error()
    status = L.fa_device_status(stream)  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert status == fa.FA_ERR_TIMEOUT, (status, L.fa_last_error())
    msg = L.fa_last_error().decode()
    m = re.search(r"site (\d+)", msg)
    assert m and 70 <= int(m.group(1)) <= 89, msg  # a wait of the pair kernel
    # 1 ms wait bound, 20 ms hand-back bound in this build: well under a second
    assert elapsed < 1.0, elapsed
    assert L.fa_device_status(stream) == fa.FA_OK

    # the context is intact: the product library's d = 256 backward meets parity
    dq, dk, dv = fa.backward(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], True, s)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == fa.FA_OK
    O, Lr = attention_forward(f64["q"], f64["k"], f64["v"], True, s)
    assert_fwd(to_np(o), O, to_np(lse), Lr, "d=256 after the starved pair")
    g = attention_backward(f64["q"], f64["k"], f64["v"], O, Lr, f64["do"], True, s)
    assert_bwd(tuple(to_np(t) for t in (dq, dk, dv)), g, "d=256 after the starved pair")
