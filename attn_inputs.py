"""Seeded synthetic inputs for exact attention (shared by the tests, the bench and the oracle checks).

This module draws random numbers and rounds them to bfloat16; it holds none of the attention
arithmetic.  Every tensor is produced by ``numpy.random.default_rng([seed, tensor_id])`` with
``tensor_id`` Q=0, K=1, V=2, dO=3, as ``standard_normal(float32) * sigma``, then rounded to
bfloat16 with round-to-nearest-even by bit manipulation.  The same uint16 bit patterns are handed
to the GPU path (as torch.bfloat16) and, widened exactly, to the fp64 oracle.

The workload shapes follow the pages' workloads: GPT-2-small (B=8, H=12, N=1024, d=64, causal),
BERT-large (B=16, H=16, N=512, d=64), long context (B=2, H=16, N=8192, d=128, causal) and a
B*H*N = 131072 sweep; the pages name no dataset, so these are shapes only.
"""
from __future__ import annotations

import numpy as np

TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "do": 3}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even); return the uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns exactly to float64."""
    u = bits.astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def draw_bits(shape, seed: int, tensor: str, sigma: float = 1.0) -> np.ndarray:
    """One seeded tensor as bfloat16 bits: N(0, sigma^2) drawn in float32, rounded to bf16."""
    rng = np.random.default_rng([int(seed), TENSOR_IDS[tensor]])
    x = rng.standard_normal(size=tuple(shape), dtype=np.float32)
    if sigma != 1.0:
        x = (x * np.float32(sigma)).astype(np.float32)
    return f32_to_bf16_bits(x)


def make_inputs(B: int, H: int, N: int, d: int, seed: int = 0, sigma_qk: float = 1.0,
                with_do: bool = True, kv_heads: int | None = None) -> dict:
    """Q, K, V (and dO) as bf16 bit arrays: Q and dO [B, H, N, d], K and V [B, H_kv, N, d] with
    H_kv = ``kv_heads`` (default H; a divisor of H for grouped-query attention).

    ``sigma_qk`` = 3 gives the peaky-softmax variant (Q, K ~ N(0, 3^2)); V and dO stay N(0, 1).
    """
    shape = (B, H, N, d)
    kv_shape = (B, H if kv_heads is None else kv_heads, N, d)
    out = {
        "q": draw_bits(shape, seed, "q", sigma_qk),
        "k": draw_bits(kv_shape, seed, "k", sigma_qk),
        "v": draw_bits(kv_shape, seed, "v", 1.0),
    }
    if with_do:
        out["do"] = draw_bits(shape, seed, "do", 1.0)
    return out


# ------------------------------------------------------------------------------------ e4m3 codes
E4M3_MAX = 448.0


def e4m3_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen e4m3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no infinities,
    S.1111.111 is NaN) exactly to float64."""
    b = np.asarray(bits).astype(np.int64)
    e = (b >> 3) & 0xF
    m = b & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(b & 0x80, -mag, mag)


def f64_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """Round values to e4m3 codes: round to nearest, ties to even, magnitudes above 448 saturate
    to 448.  Normal numbers (>= 2^-6) have 3 mantissa bits; below 2^-6 the spacing is 2^-9."""
    x = np.asarray(x, np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    _, ex = np.frexp(a)                      # a = f * 2^ex, f in [0.5, 1): binade 2^(ex-1)
    binade = np.maximum(ex - 1, -6)          # subnormals share the 2^-6 binade's spacing
    quantum = np.exp2((binade - 3).astype(np.float64))
    r = np.minimum(np.round(a / quantum) * quantum, E4M3_MAX)  # numpy rounds halves to even
    _, er = np.frexp(r)
    normal = r >= 2.0 ** -6
    exp_field = np.where(normal, er - 1 + 7, 0)
    man = np.where(normal, r / np.exp2((er - 1).astype(np.float64)) * 8.0 - 8.0, r * 2.0 ** 9)
    code = (exp_field.astype(np.int64) << 3) | man.astype(np.int64)
    return (code | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


def draw_e4m3(shape, seed: int, tensor: str, sigma: float = 1.0):
    """One seeded tensor as e4m3 codes with a per-tensor scale: the same N(0, sigma^2) float32
    draw as ``draw_bits``, divided (in float64) by scale = float32(max|x| / 448) and rounded to
    e4m3, so the codes use the whole e4m3 range.  Returns (codes uint8, scale); the tensor the
    codes stand for is scale * e4m3_bits_to_f64(codes)."""
    rng = np.random.default_rng([int(seed), TENSOR_IDS[tensor]])
    x = rng.standard_normal(size=tuple(shape), dtype=np.float32)
    if sigma != 1.0:
        x = (x * np.float32(sigma)).astype(np.float32)
    scale = float(np.float32(np.abs(x).max() / E4M3_MAX)) if x.size else 1.0
    return f64_to_e4m3_bits(x.astype(np.float64) / scale), scale


def make_inputs_fp8(B: int, H: int, N: int, d: int, seed: int = 0, sigma_qk: float = 1.0) -> dict:
    """Q, K, V [B, H, N, d] as e4m3 codes with one scale per tensor: {"q": (codes, scale), ...}.
    ``sigma_qk`` = 3 gives the peaky-softmax variant, as for ``make_inputs``."""
    shape = (B, H, N, d)
    return {"q": draw_e4m3(shape, seed, "q", sigma_qk), "k": draw_e4m3(shape, seed, "k", sigma_qk),
            "v": draw_e4m3(shape, seed, "v", 1.0)}


def default_scale(d: int) -> float:
    """The scale the workloads use, 1/sqrt(d), as a float32 value."""
    return float(np.float32(1.0 / np.sqrt(np.float64(d))))


# Named workloads (shapes from the pages' examples; see the module docstring).
WORKLOADS = {
    "tiny_fwd": dict(B=1, H=2, N=128, d=64, causal=False, fwd_only=True),
    "gpt2_small_causal": dict(B=8, H=12, N=1024, d=64, causal=True),
    "bert_large": dict(B=16, H=16, N=512, d=64, causal=False),
    "bert_large_peaky": dict(B=16, H=16, N=512, d=64, causal=False, sigma_qk=3.0),
    "long_ctx_causal": dict(B=2, H=16, N=8192, d=128, causal=True),
}


def sweep_points():
    """The B*H*N = 131072 sweep: (B, H, N) splits x d in {64,128,256} x {causal, not}."""
    splits = [(16, 16, 512), (4, 16, 2048), (1, 16, 8192), (1, 4, 32768), (1, 2, 65536)]
    pts = []
    for (B, H, N) in splits:
        for d in (64, 128, 256):
            for causal in (True, False):
                pts.append(dict(B=B, H=H, N=N, d=d, causal=causal))
    return pts
