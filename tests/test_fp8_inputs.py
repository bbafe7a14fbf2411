"""The e4m3 input path of the FP8 forward, without a GPU.

The FP8 forward attends to q_scale*Q8, k_scale*K8, v_scale*V8; its oracle is the fp64 definition
(oracle.attention_forward, pinned in test_oracle.py) on those dequantised values.  What is new
here is the e4m3 code <-> value map in attn_inputs, which both sides rely on, so it is pinned
against hand-worked codes and against torch's float8_e4m3fn conversion (an independent library
routine), and a hand-worked FP8 golden case pins the dequantisation with its three scales.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import attn_inputs as ai
from oracle import attention_forward

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_e4m3_hand_worked_codes():
    # 0x38 = 1 (exponent field 7 = bias), 0x7E = 1.75 * 2^8 = 448 (the largest finite value),
    # 0x08 = 2^-6 (smallest normal), 0x01 = 2^-9 (smallest subnormal), 0xC0 = -2
    codes = np.array([0x38, 0x7E, 0x08, 0x01, 0xC0, 0x00, 0x80], np.uint8)
    want = [1.0, 448.0, 2.0 ** -6, 2.0 ** -9, -2.0, 0.0, -0.0]
    got = ai.e4m3_bits_to_f64(codes)
    assert list(got) == want and np.signbit(got[-1])
    assert np.isnan(ai.e4m3_bits_to_f64(np.array([0x7F, 0xFF], np.uint8))).all()
    assert list(ai.f64_to_e4m3_bits(np.array(want))) == list(codes)


def test_e4m3_decode_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    mine = ai.e4m3_bits_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])


def test_e4m3_encode_matches_torch_rounding():
    """Round to nearest even on random values of every scale and on every midpoint between two
    neighbouring codes; magnitudes above 448 saturate (torch would give NaN there)."""
    vals = ai.e4m3_bits_to_f64(np.arange(0x7F, dtype=np.uint8))
    mids = (vals[:-1] + vals[1:]) / 2
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(50000) * 40, rng.standard_normal(50000) * 0.02,
                        mids, -mids, vals])
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ai.f64_to_e4m3_bits(x), ref)
    assert list(ai.f64_to_e4m3_bits(np.array([449.0, 1e6, -500.0]))) == [0x7E, 0x7E, 0xFE]


def test_fp8_inputs_use_the_range_and_round_trip():
    x = ai.make_inputs_fp8(1, 2, 64, 64, seed=3)
    for name, (codes, s) in x.items():
        vals = ai.e4m3_bits_to_f64(codes)
        assert np.abs(vals).max() == 448.0            # the largest |x| maps to 448 exactly
        assert codes.dtype == np.uint8 and codes.shape == (1, 2, 64, 64)
        # the codes stand for the float32 draw to within e4m3 rounding (2^-4 relative, or 2^-10
        # absolute for the subnormals), after the per-tensor scale
        rng = np.random.default_rng([3, ai.TENSOR_IDS[name]])
        raw = rng.standard_normal(size=(1, 2, 64, 64), dtype=np.float32).astype(np.float64)
        err = np.abs(vals * s - raw)
        assert (err <= np.maximum(np.abs(raw) * 2.0 ** -4, 2.0 ** -10 * s) * (1 + 1e-12)).all()


def _ev(x):
    return float(eval(x, {"log": math.log})) if isinstance(x, str) else float(x)


def test_fp8_golden_hand_worked():
    g = json.load(open(os.path.join(GOLDEN, "tiny_fp8_n2_d1.json")))
    deq = {t: g[f"{t}_scale"] * ai.e4m3_bits_to_f64(np.array(g[f"{t}_codes"], np.uint8))
           for t in ("q", "k", "v")}
    for t in ("q", "k", "v"):
        assert np.array_equal(deq[t], np.array(g[t], np.float64)), t
    O, L = attention_forward(*(deq[t][None, None] for t in ("q", "k", "v")), g["causal"],
                             _ev(g["scale"]))
    np.testing.assert_allclose(O[0, 0, :, 0], [_ev(r[0]) for r in g["O"]], rtol=0, atol=1e-14)
    np.testing.assert_allclose(L[0, 0], [_ev(x) for x in g["L"]], rtol=0, atol=1e-14)
    # a dequantisation that forgets q_scale gives another answer (row 1: P = [1/10, 9/10])
    bad_q = ai.e4m3_bits_to_f64(np.array(g["q_codes"], np.uint8))
    Ob, _ = attention_forward(bad_q[None, None], deq["k"][None, None], deq["v"][None, None],
                              False, _ev(g["scale"]))
    assert abs(Ob[0, 0, 1, 0] - 5.6) < 1e-12
