"""The torch conveniences of the binding validate their tensors on the host, before any launch:
wrong device, dtype, layout or head grouping raises ValueError (no GPU needed)."""
import pytest
import torch

import exact_io_aware_43_b200 as fa


def t(*shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype)


def test_forward_rejects_host_tensors():
    with pytest.raises(ValueError):
        fa.forward(t(1, 2, 8, 64), t(1, 2, 8, 64), t(1, 2, 8, 64))


def test_forward_rejects_non_dividing_kv_heads():
    with pytest.raises(ValueError):
        fa.forward(t(1, 4, 8, 64), t(1, 3, 8, 64), t(1, 3, 8, 64))


def test_forward_rejects_mismatched_lengths():
    with pytest.raises(ValueError):
        fa.forward(t(1, 2, 8, 64), t(1, 2, 9, 64), t(1, 2, 9, 64))


def test_backward_rejects_wrong_dtype():
    q = t(1, 2, 8, 64)
    with pytest.raises(ValueError):
        fa.backward(q, q, q, q, t(1, 2, 8, dtype=torch.float16), q)


def test_forward_rejects_non_4d():
    with pytest.raises(ValueError):
        fa.forward(t(2, 8, 64), t(2, 8, 64), t(2, 8, 64))


def test_splitkv_rejects_bad_kv_shape():
    with pytest.raises(ValueError):
        fa.forward_splitkv(t(1, 4, 1, 64), t(1, 3, 100, 64), t(1, 3, 100, 64))


def test_host_pipeline_rejects_wrong_shapes_and_dtypes():
    q = t(1, 2, 8, 64)
    with pytest.raises(ValueError):
        fa.forward_backward_host(q, q, q, t(1, 2, 8, 32))
    with pytest.raises(ValueError):
        fa.forward_backward_host(q, q, q, t(1, 2, 8, 64, dtype=torch.float32))


def test_kernel_names_cover_every_timer_kind():
    assert set(fa.KERNEL_NAMES) == {fa.FA_KERNEL_FWD, fa.FA_KERNEL_BWD_PRE, fa.FA_KERNEL_BWD_MAIN,
                                    fa.FA_KERNEL_BWD_POST, fa.FA_KERNEL_FWD_MERGE}
