"""exact_io_aware_43_b200 -- exact, IO-aware attention on B200 (sm_100a).

Thin Python binding over the C ABI of ``libfattn.so`` (include/fattn.h).  The functions
``fa_fwd``, ``fa_bwd``, ``fa_fwd_gqa``, ``fa_bwd_gqa``, ``fa_bwd_workspace_size``,
``fa_last_error``, ``fa_device_status`` (and the rest) have the same names and arguments as the
C entry points (pointers as Python ints, streams as raw
``cudaStream_t`` handles).  ``forward``/``backward``/``attention`` are conveniences that take
torch tensors, allocate the outputs with torch (device memory and streams are the only things
torch provides here) and call the same entry points.  There is no other code path: if the
library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "lib", "libfattn.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "fattn.h")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_MISALIGNED, FA_ERR_CUDA, \
    FA_ERR_TIMEOUT, FA_ERR_WORKSPACE = range(7)

_lib = None


class FattnError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libfattn error {code}: {msg}")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libfattn.so (built in-tree by ``python -m exact_io_aware_43_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise FattnError(-1, f"{LIB_PATH} is missing; build it with "
                             "`python -m exact_io_aware_43_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
    L.fa_fwd.restype = i
    L.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    L.fa_bwd_workspace_size.restype = sz
    L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, sz, vp]
    L.fa_bwd.restype = i
    L.fa_bwd_gqa_workspace_size.argtypes = [i, i, i, i, i]
    L.fa_bwd_gqa_workspace_size.restype = sz
    L.fa_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp]
    L.fa_fwd_gqa.restype = i
    L.fa_bwd_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp, sz, vp]
    L.fa_bwd_gqa.restype = i
    L.fa_fwd_splitkv_workspace_size.argtypes = [i, i, i, i, i, i]
    L.fa_fwd_splitkv_workspace_size.restype = sz
    L.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, vp, sz, vp]
    L.fa_fwd_splitkv.restype = i
    L.fa_fwd_bwd_host_device_bytes.argtypes = [i, i, i, i, i]
    L.fa_fwd_bwd_host_device_bytes.restype = sz
    L.fa_fwd_bwd_host.argtypes = [vp] * 9 + [i, i, i, i, i, f, i, vp, sz, vp]
    L.fa_fwd_bwd_host.restype = i
    L.fa_last_error.argtypes = []
    L.fa_last_error.restype = ctypes.c_char_p
    L.fa_device_status.argtypes = [vp]
    L.fa_device_status.restype = i
    L.fa_version.argtypes = []
    L.fa_version.restype = i
    L.fa_fwd_fp8.argtypes = [vp, vp, vp, f, f, f, vp, vp, i, i, i, i, i, f, vp]
    L.fa_fwd_fp8.restype = i
    L.fa_fwd_partial.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, vp]
    L.fa_fwd_partial.restype = i
    L.fa_merge_partials.argtypes = [vp, vp, i, vp, vp, ctypes.c_longlong, i, vp]
    L.fa_merge_partials.restype = i
    L.fa_selftest_exp2_fma.argtypes = [vp, vp, i, vp]
    L.fa_selftest_exp2_fma.restype = i
    L.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
    L.fa_bwd_noalloc.restype = i
    L.fa_timer_enable.argtypes = [i]
    L.fa_timer_enable.restype = i
    L.fa_timer_read.argtypes = [i, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]
    L.fa_timer_read.restype = i
    _lib = L
    return L


def header_functions() -> list[str]:
    """Names of the functions include/fattn.h declares."""
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(fa_\w+)\s*\(", txt, flags=re.M)


# ------------------------------------------------------------------ C entry points, same names
def fa_last_error() -> str:
    return lib().fa_last_error().decode()


def _check(rc: int) -> int:
    if rc != FA_OK:
        raise FattnError(rc, fa_last_error())
    return rc


def fa_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, stream) -> int:
    return lib().fa_fwd(q, k, v, o, lse, B, H, N, d, int(causal), float(scale), stream)


def fa_bwd_workspace_size(B, H, N, d) -> int:
    return lib().fa_bwd_workspace_size(B, H, N, d)


def fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, causal, scale, workspace,
           workspace_bytes, stream) -> int:
    return lib().fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, int(causal), float(scale),
                        workspace, workspace_bytes, stream)


def fa_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B, H, N, d, causal, scale,
               stream) -> int:
    return lib().fa_fwd_fp8(q8, k8, v8, float(q_scale), float(k_scale), float(v_scale), o, lse,
                            B, H, N, d, int(causal), float(scale), stream)


def fa_fwd_partial(q, k, v, o_part, lse_part, B, H, H_kv, Nq, Nk, d, causal, scale,
                   stream) -> int:
    return lib().fa_fwd_partial(q, k, v, o_part, lse_part, B, H, H_kv, Nq, Nk, d, int(causal),
                                float(scale), stream)


def fa_merge_partials(o_parts, lse_parts, n_parts, o, lse, rows, d, stream) -> int:
    return lib().fa_merge_partials(o_parts, lse_parts, n_parts, o, lse, rows, d, stream)


def fa_selftest_exp2_fma(x, y, n, stream) -> int:
    return lib().fa_selftest_exp2_fma(x, y, n, stream)


def fa_bwd_gqa_workspace_size(B, H, H_kv, N, d) -> int:
    return lib().fa_bwd_gqa_workspace_size(B, H, H_kv, N, d)


def fa_fwd_gqa(q, k, v, o, lse, B, H, H_kv, N, d, causal, scale, stream) -> int:
    return lib().fa_fwd_gqa(q, k, v, o, lse, B, H, H_kv, N, d, int(causal), float(scale), stream)


def fa_bwd_gqa(q, k, v, o, lse, dO, dq, dk, dv, B, H, H_kv, N, d, causal, scale, workspace,
               workspace_bytes, stream) -> int:
    return lib().fa_bwd_gqa(q, k, v, o, lse, dO, dq, dk, dv, B, H, H_kv, N, d, int(causal),
                            float(scale), workspace, workspace_bytes, stream)


def fa_fwd_splitkv_workspace_size(B, H, Nq, Nk, d, splits) -> int:
    return lib().fa_fwd_splitkv_workspace_size(B, H, Nq, Nk, d, splits)


def fa_fwd_splitkv(q, k, v, o, lse, B, H, H_kv, Nq, Nk, d, causal, scale, splits, workspace,
                   workspace_bytes, stream) -> int:
    return lib().fa_fwd_splitkv(q, k, v, o, lse, B, H, H_kv, Nq, Nk, d, int(causal), float(scale),
                                int(splits), workspace, workspace_bytes, stream)


def fa_fwd_bwd_host_device_bytes(B, H, N, d, chunks) -> int:
    return lib().fa_fwd_bwd_host_device_bytes(B, H, N, d, chunks)


def fa_fwd_bwd_host(q, k, v, dO, o, lse, dq, dk, dv, B, H, N, d, causal, scale, chunks,
                    device_buffer, device_bytes, stream) -> int:
    return lib().fa_fwd_bwd_host(q, k, v, dO, o, lse, dq, dk, dv, B, H, N, d, int(causal),
                                 float(scale), int(chunks), device_buffer, device_bytes, stream)


def fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, causal, scale, stream) -> int:
    """fa_bwd with the library's static scratch instead of a caller workspace (for callers that
    cannot allocate device memory; shapes up to FA_NOALLOC_SCRATCH_BYTES of workspace)."""
    return lib().fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, int(causal),
                                float(scale), stream)


FA_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def fa_device_status(stream=None) -> int:
    return lib().fa_device_status(stream)


def fa_version() -> int:
    return lib().fa_version()


FA_KERNEL_FWD, FA_KERNEL_BWD_PRE, FA_KERNEL_BWD_MAIN, FA_KERNEL_BWD_POST, FA_KERNEL_FWD_MERGE = range(5)
KERNEL_NAMES = {FA_KERNEL_FWD: "fa_fwd_kernel", FA_KERNEL_BWD_PRE: "fa_bwd_pre_kernel",
                FA_KERNEL_BWD_MAIN: "fa_bwd_kernel", FA_KERNEL_BWD_POST: "fa_bwd_post_kernel",
                FA_KERNEL_FWD_MERGE: "fa_fwd_merge_kernel"}


def fa_timer_enable(on: bool) -> int:
    return lib().fa_timer_enable(int(bool(on)))


def fa_timer_read(kernel: int):
    """(launches, total_ms) recorded for one kernel kind since the last read."""
    n = ctypes.c_int(0)
    ms = ctypes.c_double(0.0)
    _check(lib().fa_timer_read(kernel, ctypes.byref(n), ctypes.byref(ms)))
    return n.value, ms.value


# ------------------------------------------------------------------ torch conveniences
def _stream_handle(t):
    import torch
    return torch.cuda.current_stream(t.device).cuda_stream


def _shape(q):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(q.shape)


def _default_scale(d):
    import numpy as np
    return float(np.float32(1.0 / np.sqrt(np.float64(d))))


def _check_tensor(t, shape, dtype, name):
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != shape:
        raise ValueError(f"{name} must be a contiguous {dtype} CUDA tensor of shape {shape}")


def _kv_heads(q, k):
    """H_kv of k ([B, H_kv, N, d]); H_kv must divide q's H (grouped-query attention)."""
    B, H, N, d = _shape(q)
    if k.dim() != 4 or k.shape[0] != B or k.shape[2] != N or k.shape[3] != d or \
            k.shape[1] < 1 or H % k.shape[1] != 0:
        raise ValueError("k, v must be [B, H_kv, N, d] with H_kv dividing q's H")
    return int(k.shape[1])


def forward(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None):
    """O, L = attention(q, k, v) for contiguous bf16 CUDA tensors: q [B, H, N, d] and k, v
    [B, H_kv, N, d] (H_kv = H, or a divisor of H for grouped-query attention)."""
    import torch
    B, H, N, d = _shape(q)
    Hkv = _kv_heads(q, k)
    _check_tensor(q, (B, H, N, d), torch.bfloat16, "q")
    _check_tensor(k, (B, Hkv, N, d), torch.bfloat16, "k")
    _check_tensor(v, (B, Hkv, N, d), torch.bfloat16, "v")
    scale = _default_scale(d) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    L = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor(o, (B, H, N, d), torch.bfloat16, "out")
    _check_tensor(L, (B, H, N), torch.float32, "lse")
    if Hkv == H:
        rc = fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), L.data_ptr(),
                    B, H, N, d, causal, scale, _stream_handle(q))
    else:
        rc = fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), L.data_ptr(),
                        B, H, Hkv, N, d, causal, scale, _stream_handle(q))
    _check(rc)
    return o, L


def backward(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None,
             workspace=None, grads=None):
    """dQ, dK, dV for contiguous bf16 CUDA tensors; ``workspace`` (uint8 CUDA tensor) optional."""
    import torch
    B, H, N, d = _shape(q)
    Hkv = _kv_heads(q, k)
    for t, shp, name in ((q, (B, H, N, d), "q"), (k, (B, Hkv, N, d), "k"),
                         (v, (B, Hkv, N, d), "v"), (o, (B, H, N, d), "o"),
                         (do, (B, H, N, d), "do")):
        _check_tensor(t, shp, torch.bfloat16, name)
    _check_tensor(lse, (B, H, N), torch.float32, "lse")
    scale = _default_scale(d) if scale is None else float(scale)
    need = fa_bwd_gqa_workspace_size(B, H, Hkv, N, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    dq, dk, dv = grads
    for t, shp, name in ((dq, (B, H, N, d), "dq"), (dk, (B, Hkv, N, d), "dk"),
                         (dv, (B, Hkv, N, d), "dv")):
        _check_tensor(t, shp, torch.bfloat16, name)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
            do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr())
    if Hkv == H:
        rc = fa_bwd(*args, B, H, N, d, causal, scale, workspace.data_ptr(), workspace.numel(),
                    _stream_handle(q))
    else:
        rc = fa_bwd_gqa(*args, B, H, Hkv, N, d, causal, scale, workspace.data_ptr(),
                        workspace.numel(), _stream_handle(q))
    _check(rc)
    return dq, dk, dv


def forward_fp8(q8, k8, v8, q_scale: float, k_scale: float, v_scale: float,
                causal: bool = False, scale: float | None = None, out=None, lse=None):
    """O, L = attention(q_scale*Q8, k_scale*K8, v_scale*V8) for e4m3 code tensors q8, k8, v8
    (contiguous CUDA tensors of dtype uint8 or float8_e4m3fn, [B, H, N, d]); O is bf16, L fp32."""
    import torch
    B, H, N, d = _shape(q8)
    for t, name in ((q8, "q8"), (k8, "k8"), (v8, "v8")):
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn) or not t.is_cuda or \
                not t.is_contiguous() or tuple(t.shape) != (B, H, N, d):
            raise ValueError(f"{name} must be a contiguous uint8/float8_e4m3fn CUDA tensor of "
                             f"shape {(B, H, N, d)}")
    scale = _default_scale(d) if scale is None else float(scale)
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device) if out is None else out
    L = torch.empty((B, H, N), dtype=torch.float32, device=q8.device) if lse is None else lse
    _check_tensor(o, (B, H, N, d), torch.bfloat16, "out")
    _check_tensor(L, (B, H, N), torch.float32, "lse")
    _check(fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), q_scale, k_scale, v_scale,
                      o.data_ptr(), L.data_ptr(), B, H, N, d, causal, scale, _stream_handle(q8)))
    return o, L


def default_splits(B, H, Nq, Nk, device=None, H_kv=None) -> int:
    """A split count for fa_fwd_splitkv: one range when (query blocks x heads) already give about
    one work unit per SM, else about two units per SM (at most one range per 128-key tile).  With
    grouped heads and G * Nq <= 128 one unit serves a whole group (packed query heads).  Measured
    on B=16 H=32 H_kv=8 Nq=1 Nk=8192 d=128: 1 range 3888 GB/s, 2: 3570, 4: 3503, 8: 3692."""
    import torch
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    G = H // H_kv if H_kv else 1
    if G > 1 and G * Nq <= 128:
        units = B * (H // G)
    else:
        units = B * H * ((Nq + 255) // 256)
    tiles = (Nk + 127) // 128
    if 4 * units >= 3 * sms:
        return 1  # the units nearly fill the GPU: a merge would cost more than it saves
    return max(1, min(tiles, (2 * sms + units - 1) // units))


def forward_splitkv(q, k, v, causal: bool = False, scale: float | None = None,
                    splits: int | None = None, out=None, lse=None, workspace=None):
    """O, L for q [B, H, Nq, d] against k, v [B, H_kv, Nk, d] (Nq and Nk may differ; causal is
    aligned to the end of the keys) with the keys split into ``splits`` ranges and merged."""
    import torch
    B, H, Nq, d = _shape(q)
    if k.dim() != 4 or k.shape[0] != B or k.shape[3] != d or k.shape[1] < 1 or H % k.shape[1]:
        raise ValueError("k, v must be [B, H_kv, Nk, d] with H_kv dividing q's H")
    Hkv, Nk = int(k.shape[1]), int(k.shape[2])
    _check_tensor(q, (B, H, Nq, d), torch.bfloat16, "q")
    _check_tensor(k, (B, Hkv, Nk, d), torch.bfloat16, "k")
    _check_tensor(v, (B, Hkv, Nk, d), torch.bfloat16, "v")
    scale = _default_scale(d) if scale is None else float(scale)
    if splits is None:
        splits = default_splits(B, H, Nq, Nk, q.device, Hkv)
    o = torch.empty_like(q) if out is None else out
    L = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check_tensor(o, (B, H, Nq, d), torch.bfloat16, "out")
    _check_tensor(L, (B, H, Nq), torch.float32, "lse")
    need = fa_fwd_splitkv_workspace_size(B, H, Nq, Nk, d, splits)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), L.data_ptr(),
                          B, H, Hkv, Nq, Nk, d, causal, scale, splits, workspace.data_ptr(),
                          workspace.numel(), _stream_handle(q)))
    return o, L


def forward_backward_host(q, k, v, do, causal: bool = False, scale: float | None = None,
                          chunks: int = 4, grads=None, out=None, lse=None, device_buffer=None,
                          stream=None):
    """fa_fwd_bwd_host on CPU tensors (pinned for overlapped copies): returns (dq, dk, dv) as
    CPU tensors; ``out`` / ``lse`` (CPU tensors) also receive O and L when given.  The call
    synchronises the stream before returning."""
    import torch
    B, H, N, d = _shape(q)
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (do, "do")):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous() or \
                tuple(t.shape) != (B, H, N, d):
            raise ValueError(f"{name} must be a contiguous bf16 CPU tensor of shape {(B, H, N, d)}")
    scale = _default_scale(d) if scale is None else float(scale)
    if grads is None:
        grads = tuple(torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory()
                      for _ in range(3))
    need = fa_fwd_bwd_host_device_bytes(B, H, N, d, chunks)
    if device_buffer is None:
        device_buffer = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream() if stream is None else stream
    _check(fa_fwd_bwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(),
                           out.data_ptr() if out is not None else None,
                           lse.data_ptr() if lse is not None else None,
                           grads[0].data_ptr(), grads[1].data_ptr(), grads[2].data_ptr(),
                           B, H, N, d, causal, scale, chunks, device_buffer.data_ptr(),
                           device_buffer.numel(), st.cuda_stream))
    st.synchronize()
    return grads


def attention(q, k, v, causal: bool = False, scale: float | None = None):
    """Differentiable attention (torch.autograd.Function over fa_fwd / fa_bwd)."""
    import torch

    class _Fn(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v):
            o, L = forward(q, k, v, causal, scale)
            ctx.save_for_backward(q, k, v, o, L)
            return o

        @staticmethod
        def backward(ctx, do):
            q, k, v, o, L = ctx.saved_tensors
            return backward(q, k, v, o, L, do.contiguous(), causal, scale)

    return _Fn.apply(q, k, v)
