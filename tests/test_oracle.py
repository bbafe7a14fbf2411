"""Pins for the fp64 oracle: it is checked against facts fixed by the pages and by mathematics,
never against itself.

Each pin is written as a function of an implementation (forward, backward) so the same pins can be
run on deliberately broken copies of the oracle (the "planted mistakes" at the end) to show that a
plausible slip -- a dropped rescale, a wrong sign, a transposed operand, a missing scale -- fails
at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import attn_inputs as ai
from oracle import (attention_backward, attention_dkdv_key_rows, attention_forward,
                    attention_forward_online, attention_probs, attention_row_stats)
from oracle.attention import _block_summary

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(shape, seed, sigma=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * sigma


# --------------------------------------------------------------------------------------------
# hand-worked fixtures


def _ev(x):
    if isinstance(x, str):
        return float(eval(x, {"log": math.log, "exp": math.exp, "sqrt": math.sqrt}))
    return float(x)


def _arr(rows):
    return np.array([[_ev(c) for c in r] if isinstance(r, list) else _ev(r) for r in rows])


GOLDEN_CASES = ["tiny_noncausal_n2_d1.json", "tiny_causal_n2_d1.json", "tiny_scaled_n2_d1.json"]


@pytest.mark.parametrize("name", GOLDEN_CASES)
def test_golden_hand_worked(name):
    g = json.load(open(os.path.join(GOLDEN, name)))
    q, k, v, do = (_arr(g[t])[None, None] for t in ("q", "k", "v", "do"))
    O, L = attention_forward(q, k, v, g["causal"], g["scale"])
    np.testing.assert_allclose(O[0, 0], _arr(g["O"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(L[0, 0], _arr(g["L"]), rtol=0, atol=1e-14)
    dq, dk, dv = attention_backward(q, k, v, O, L, do, g["causal"], g["scale"])
    np.testing.assert_allclose(dq[0, 0], _arr(g["dQ"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk[0, 0], _arr(g["dK"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv[0, 0], _arr(g["dV"]), rtol=0, atol=1e-13)


def _golden_probs_error(name, probs):
    g = json.load(open(os.path.join(GOLDEN, name)))
    q, k = (_arr(g[t])[None, None] for t in ("q", "k"))
    P = probs(q, k, g["causal"], g["scale"])
    return float(np.abs(P[0, 0] - _arr(g["P"])).max())


@pytest.mark.parametrize("name", GOLDEN_CASES)
def test_golden_probabilities(name):
    """attention_probs against the hand-worked P of each golden case."""
    assert _golden_probs_error(name, attention_probs) <= 1e-15


def test_golden_probabilities_catch_a_scale_slip():
    """A probability helper that drops (or doubles) the scale fails the scaled golden case."""
    dropped = lambda q, k, c, s: attention_probs(q, k, c, 1.0)
    doubled = lambda q, k, c, s: attention_probs(q, k, c, 2.0 * s)
    for bad in (dropped, doubled):
        assert _golden_probs_error("tiny_scaled_n2_d1.json", bad) > 1e-3


def test_golden_naive_score_bytes():
    g = json.load(open(os.path.join(GOLDEN, "naive_score_matrix_bytes.json")))
    assert g["batch_heads"] * g["N"] * g["N"] * g["bytes_per_element"] == g["bytes"]


# --------------------------------------------------------------------------------------------
# pins as functions of an implementation; each returns None when it holds, else a message


def pin_online_equals_two_pass(fwd, online):
    """[P3] 'Online Softmax Trick' and [P4] 'Softmax online': the blockwise result is identical."""
    q, k, v = (rand((1, 2, 37, 8), s) for s in (1, 2, 3))
    for causal in (False, True):
        O2, L2 = fwd(q, k, v, causal, 0.35)
        for (br, bc) in ((1, 1), (7, 7), (16, 5), (64, 64), (37, 1), (5, 37)):
            for tree in (False, True):
                O1, L1 = online(q, k, v, causal, 0.35, br, bc, tree)
                if not (np.allclose(O1, O2, atol=1e-12, rtol=0) and
                        np.allclose(L1, L2, atol=1e-12)):
                    return f"online != two-pass at causal={causal} Br={br} Bc={bc} tree={tree}"
    return None


def pin_constant_v(fwd):
    """Rows of P sum to 1, so V = c (every row the same vector) gives O = c exactly."""
    q, k = rand((2, 2, 33, 16), 4), rand((2, 2, 33, 16), 5)
    c = rand((16,), 6)
    v = np.broadcast_to(c, (2, 2, 33, 16)).copy()
    for causal in (False, True):
        O, _ = fwd(q, k, v, causal, 0.25)
        if not np.allclose(O, c, atol=1e-13, rtol=0):
            return "constant V did not give constant O"
    return None


def pin_causal_row0(fwd):
    """Causal: query 0 sees only key 0, so O_0 = V_0 and L_0 = scale * q_0 . k_0."""
    q, k, v = (rand((1, 3, 20, 8), s) for s in (7, 8, 9))
    O, L = fwd(q, k, v, True, 0.5)
    if not np.allclose(O[:, :, 0], v[:, :, 0], atol=1e-14, rtol=0):
        return "causal row 0 != V[0]"
    if not np.allclose(L[:, :, 0], 0.5 * np.sum(q[:, :, 0] * k[:, :, 0], -1), atol=1e-13):
        return "causal L_0 != s q0.k0"
    return None


def pin_zero_q(fwd):
    """Q = 0: every score is 0, so P is uniform over the visible keys.
    Non-causal: L_i = ln N and O_i = mean of V.  Causal: L_i = ln(i+1), O_i = mean of V[0..i]."""
    N = 29
    q = np.zeros((1, 2, N, 8))
    k, v = rand((1, 2, N, 8), 10), rand((1, 2, N, 8), 11)
    O, L = fwd(q, k, v, False, 0.3)
    if not (np.allclose(L, np.log(N), atol=1e-14) and
            np.allclose(O, v.mean(axis=2, keepdims=True), atol=1e-14)):
        return "Q=0 non-causal closed form"
    O, L = fwd(q, k, v, True, 0.3)
    pref = np.cumsum(v, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    if not (np.allclose(L, np.log(np.arange(1, N + 1)), atol=1e-14) and
            np.allclose(O, pref, atol=1e-13)):
        return "Q=0 causal closed form"
    return None


def pin_shift_invariance(fwd):
    """Adding one vector c to every key adds q_i . c to a whole score row: O is unchanged and
    L shifts by scale * q_i . c."""
    q, k, v = (rand((1, 2, 24, 8), s) for s in (12, 13, 14))
    c = rand((8,), 15)
    for causal in (False, True):
        O1, L1 = fwd(q, k, v, causal, 0.4)
        O2, L2 = fwd(q, k + c, v, causal, 0.4)
        if not np.allclose(O1, O2, atol=1e-12):
            return "shift of K changed O"
        if not np.allclose(L2 - L1, 0.4 * q @ c, atol=1e-12):
            return "shift of K did not shift L by s q.c"
    return None


def pin_probabilities(fwd):
    """O = P V with P row-stochastic: compare against P from softmax of the scores by hand
    (rows sum to 1, entries in [0,1], masked entries exactly 0)."""
    q, k, v = (rand((1, 1, 17, 4), s) for s in (16, 17, 18))
    for causal in (False, True):
        O, _ = fwd(q, k, v, causal, 0.7)
        # v = identity columns picks out P itself: O = P when V = I (N x N, d = N)
        eye = np.eye(17)[None, None]
        P, _ = fwd(q, k, eye, causal, 0.7)
        if not np.allclose(P.sum(-1), 1.0, atol=1e-14):
            return "rows of P do not sum to 1"
        if P.min() < 0 or P.max() > 1:
            return "P outside [0,1]"
        if causal and np.abs(np.triu(P[0, 0], 1)).max() != 0.0:
            return "masked P entries are not zero"
        if not np.allclose(P @ v, O, atol=1e-13):
            return "O != P V"
    return None


def pin_library_forward(fwd):
    """Cross-check with an independent library routine: torch's CPU float64 scaled_dot_product
    attention (math backend)."""
    q, k, v = (rand((2, 3, 40, 16), s) for s in (19, 20, 21))
    for causal in (False, True):
        O, _ = fwd(q, k, v, causal, 0.25)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
            is_causal=causal, scale=0.25).numpy()
        if not np.allclose(O, ref, atol=1e-12):
            return "forward disagrees with torch float64 SDPA"
    return None


def _loss_grad_fd(q, k, v, do, causal, scale, fwd, h=1e-6):
    """Central finite differences of loss = sum(O * dO) with respect to q, k, v."""
    grads = []
    for which in range(3):
        base = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(base[which])
        it = np.nditer(g, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [a.copy() for a in base]
            minus = [a.copy() for a in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            Op, _ = fwd(*plus, causal, scale)
            Om, _ = fwd(*minus, causal, scale)
            g[idx] = (np.sum(Op * do) - np.sum(Om * do)) / (2 * h)
        grads.append(g)
    return grads


def pin_finite_differences(fwd, bwd):
    """Brute force: the analytic backward equals central finite differences on tiny inputs."""
    for causal in (False, True):
        for (N, d, seed) in ((5, 3, 30), (8, 4, 31), (3, 2, 32)):
            q, k, v, do = (rand((1, 1, N, d), seed + 10 * i) for i in range(4))
            O, L = fwd(q, k, v, causal, 0.6)
            dq, dk, dv = bwd(q, k, v, O, L, do, causal, 0.6)
            fq, fk, fv = _loss_grad_fd(q, k, v, do, causal, 0.6, fwd)
            for a, b in ((dq, fq), (dk, fk), (dv, fv)):
                if not np.allclose(a, b, rtol=1e-6, atol=1e-8):
                    return f"analytic backward != finite differences (causal={causal}, N={N})"
    return None


def pin_library_backward(fwd, bwd):
    """Cross-check with torch float64 autograd through plain softmax attention."""
    q, k, v, do = (rand((1, 2, 33, 8), s) for s in (40, 41, 42, 43))
    for causal in (False, True):
        O, L = fwd(q, k, v, causal, 0.3)
        dq, dk, dv = bwd(q, k, v, O, L, do, causal, 0.3)
        tq, tk, tv = (torch.from_numpy(a).requires_grad_() for a in (q, k, v))
        to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal,
                                                              scale=0.3)
        to.backward(torch.from_numpy(do))
        for a, t in ((dq, tq), (dk, tk), (dv, tv)):
            if not np.allclose(a, t.grad.numpy(), atol=1e-12):
                return "backward disagrees with torch float64 autograd"
    return None


def pin_backward_invariants(fwd, bwd):
    """Rows of P sum to 1, hence sum_j dS_ij = 0, hence sum_j dK_j = 0; and
    sum_j dV_j = sum_i dO_i (per head)."""
    q, k, v, do = (rand((2, 2, 31, 8), s) for s in (50, 51, 52, 53))
    for causal in (False, True):
        O, L = fwd(q, k, v, causal, 0.4)
        dq, dk, dv = bwd(q, k, v, O, L, do, causal, 0.4)
        if not np.allclose(dk.sum(axis=2), 0.0, atol=1e-12):
            return "sum_j dK_j != 0"
        if not np.allclose(dv.sum(axis=2), do.sum(axis=2), atol=1e-12):
            return "sum_j dV_j != sum_i dO_i"
    return None


def pin_peaky(fwd):
    """Scaled scores with std ~9 (Q, K ~ N(0, 3^2), d = 64): without the max subtraction exp
    overflows in fp32; the result must stay finite and row-stochastic."""
    q, k = rand((1, 1, 64, 64), 60, 3.0), rand((1, 1, 64, 64), 61, 3.0) * 3.0
    v = np.eye(64)[None, None]
    P, L = fwd(q, k, v, False, 0.125)
    if not (np.isfinite(P).all() and np.isfinite(L).all()):
        return "peaky softmax not finite"
    if not np.allclose(P.sum(-1), 1.0, atol=1e-13):
        return "peaky softmax rows do not sum to 1"
    return None


FWD_PINS = [pin_constant_v, pin_causal_row0, pin_zero_q, pin_shift_invariance, pin_probabilities,
            pin_library_forward, pin_peaky]
BWD_PINS = [pin_finite_differences, pin_library_backward, pin_backward_invariants]


def run_pins(fwd, online, bwd):
    fails = []
    for p in FWD_PINS:
        m = p(fwd)
        if m:
            fails.append(m)
    m = pin_online_equals_two_pass(fwd, online)
    if m:
        fails.append(m)
    for p in BWD_PINS:
        m = p(fwd, bwd)
        if m:
            fails.append(m)
    return fails


@pytest.mark.parametrize("pin", FWD_PINS, ids=lambda p: p.__name__)
def test_forward_pin(pin):
    assert pin(attention_forward) is None


@pytest.mark.parametrize("pin", BWD_PINS, ids=lambda p: p.__name__)
def test_backward_pin(pin):
    assert pin(attention_forward, attention_backward) is None


def test_online_equals_two_pass():
    assert pin_online_equals_two_pass(attention_forward, attention_forward_online) is None


def test_online_forward_pins():
    """The tiled (online) forward meets the forward pins as well."""
    online = lambda q, k, v, c, s: attention_forward_online(q, k, v, c, s, 8, 5)
    for p in FWD_PINS:
        assert p(online) is None, p.__name__


def test_probs_helper_rows():
    q, k = rand((1, 2, 12, 4), 70), rand((1, 2, 12, 4), 71)
    P = attention_probs(q, k, True, 0.5)
    assert np.allclose(P.sum(-1), 1.0, atol=1e-14)
    assert np.all(np.triu(P[0, 0], 1) == 0)


def test_oracle_on_bf16_inputs_tiny_workload():
    """The oracle runs on the exactly widened bf16 inputs of the smallest workload (B=1, H=2,
    N=128, d=64) and agrees with torch's float64 SDPA there."""
    w = ai.WORKLOADS["tiny_fwd"]
    x = ai.make_inputs(w["B"], w["H"], w["N"], w["d"], seed=0, with_do=False)
    q, k, v = (ai.bf16_bits_to_f64(x[t]) for t in ("q", "k", "v"))
    s = ai.default_scale(w["d"])
    O, L = attention_forward(q, k, v, False, s)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), scale=s).numpy()
    assert np.allclose(O, ref, atol=1e-12)
    assert np.isfinite(L).all()


# --------------------------------------------------------------------------------------------
# planted mistakes: broken copies of the oracle must fail at least one pin


def _mut_fwd_no_max(q, k, v, causal, scale):
    # forgets the max subtraction in L (uses ln l only)
    O, L = attention_forward(q, k, v, causal, scale)
    S = np.einsum("bhnd,bhmd->bhnm", q, k) * scale
    if causal:
        S = np.where(np.triu(np.ones(S.shape[-2:]), 1) > 0, -np.inf, S)
    return O, L - S.max(-1)


def _mut_fwd_unscaled(q, k, v, causal, scale):
    return attention_forward(q, k, v, causal, 1.0)


def _mut_fwd_causal_off_by_one(q, k, v, causal, scale):
    # mask keeps j < i instead of j <= i (row 0 then has no key; use j <= i+1 instead)
    q = np.asarray(q, np.float64)
    B, H, N, d = q.shape
    O = np.empty((B, H, N, v.shape[-1]))
    L = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            s = scale * q[b, h] @ k[b, h].T
            if causal:
                s[np.triu_indices(N, 2)] = -np.inf
            m = s.max(1, keepdims=True)
            e = np.exp(s - m)
            O[b, h] = e / e.sum(1, keepdims=True) @ v[b, h]
            L[b, h] = (m + np.log(e.sum(1, keepdims=True)))[:, 0]
    return O, L


def _mut_online_no_rescale(q, k, v, causal, scale, br, bc, tree=False):
    # merges block summaries without moving the running output onto the new maximum
    q = np.asarray(q, np.float64)
    B, H, N, d = q.shape
    O = np.empty((B, H, N, v.shape[-1]))
    L = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, br):
                r1 = min(N, r0 + br)
                m = np.full(r1 - r0, -np.inf)
                l = np.zeros(r1 - r0)
                u = np.zeros((r1 - r0, v.shape[-1]))
                for c0 in range(0, N, bc):
                    c1 = min(N, c0 + bc)
                    s = scale * q[b, h, r0:r1] @ k[b, h, c0:c1].T
                    if causal:
                        s = np.where(np.arange(c0, c1)[None] > np.arange(r0, r1)[:, None],
                                     -np.inf, s)
                    m2, l2, u2 = _block_summary(s, v[b, h, c0:c1])
                    mn = np.maximum(m, m2)
                    ref = np.where(np.isfinite(mn), mn, 0.0)
                    w1 = np.where(np.isfinite(m), np.exp(m - ref), 0.0)
                    w2 = np.where(np.isfinite(m2), np.exp(m2 - ref), 0.0)
                    l = w1 * l + w2 * l2
                    u = u + w2[:, None] * u2  # the slip: u is not multiplied by w1
                    m = mn
                O[b, h, r0:r1] = u / l[:, None]
                L[b, h, r0:r1] = m + np.log(l)
    return O, L


def _mut_bwd_sign(q, k, v, o, lse, do, causal, scale):
    # dS = P * (D - dP) instead of P * (dP - D), seen through dK only
    dq, dk, dv = attention_backward(q, k, v, o, lse, do, causal, scale)
    return dq, -dk, dv


def _mut_bwd_no_D(q, k, v, o, lse, do, causal, scale):
    # forgets the D = rowsum(dO * O) term: pass O = 0
    return attention_backward(q, k, v, np.zeros_like(o), lse, do, causal, scale)


def _mut_bwd_transposed_dv(q, k, v, o, lse, do, causal, scale):
    # dV = P dO instead of P^T dO
    dq, dk, dv = attention_backward(q, k, v, o, lse, do, causal, scale)
    P = attention_probs(q, k, causal, scale)
    return dq, dk, np.einsum("bhij,bhjd->bhid", P, do)


def _mut_bwd_missing_scale(q, k, v, o, lse, do, causal, scale):
    dq, dk, dv = attention_backward(q, k, v, o, lse, do, causal, scale)
    return dq / scale, dk, dv


MUTANTS = [
    ("fwd_L_without_max", _mut_fwd_no_max, None, None),
    ("fwd_unscaled", _mut_fwd_unscaled, None, None),
    ("fwd_causal_off_by_one", _mut_fwd_causal_off_by_one, None, None),
    ("online_no_rescale", None, _mut_online_no_rescale, None),
    ("bwd_sign_dk", None, None, _mut_bwd_sign),
    ("bwd_no_D", None, None, _mut_bwd_no_D),
    ("bwd_transposed_dv", None, None, _mut_bwd_transposed_dv),
    ("bwd_missing_scale_dq", None, None, _mut_bwd_missing_scale),
]


@pytest.mark.parametrize("name,fwd,online,bwd", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, fwd, online, bwd):
    fails = run_pins(fwd or attention_forward, online or attention_forward_online,
                     bwd or attention_backward)
    assert fails, f"planted mistake {name} passed every pin"


def test_oracle_passes_all_pins():
    assert run_pins(attention_forward, attention_forward_online, attention_backward) == []


# --------------------------------------------------------------------------------------------
# row-sampled oracle functions (used where a head is too long for the full N x N oracle)


@pytest.mark.parametrize("causal", [False, True])
def test_rows_match_full_oracle(causal):
    q, k, v, do = (rand((1, 1, 45, 8), s) for s in (80, 81, 82, 83))
    O, L = attention_forward(q, k, v, causal, 0.3)
    dq, _, _ = attention_backward(q, k, v, O, L, do, causal, 0.3)
    rows = np.array([0, 1, 7, 30, 44])
    Or, Lr = __import__("oracle").attention_rows(q[0, 0], k[0, 0], v[0, 0], rows, causal, 0.3)
    dqr = __import__("oracle").attention_dq_rows(q[0, 0], k[0, 0], v[0, 0], do[0, 0], rows, causal,
                                               0.3)
    assert np.allclose(Or, O[0, 0, rows], atol=1e-13) and np.allclose(Lr, L[0, 0, rows], atol=1e-13)
    assert np.allclose(dqr, dq[0, 0, rows], atol=1e-12)


def test_rows_closed_forms():
    """Q = 0 rows: L = ln(i+1) causal, O = prefix mean; dQ of row 0 (causal) is exactly 0."""
    import oracle as orc
    N = 33
    q = np.zeros((N, 4))
    k, v, do = rand((N, 4), 84), rand((N, 4), 85), rand((N, 4), 86)
    rows = np.array([0, 5, 32])
    O, L = orc.attention_rows(q, k, v, rows, True, 0.5)
    assert np.allclose(L, np.log(rows + 1), atol=1e-14)
    assert np.allclose(O, np.stack([v[:r + 1].mean(0) for r in rows]), atol=1e-14)
    dq = orc.attention_dq_rows(rand((N, 4), 87), k, v, do, np.array([0]), True, 0.5)
    assert np.allclose(dq, 0.0, atol=1e-15)


# --------------------------------------------------------------------------------------------
# key-row gradients (used where a head is too long for the full N x N oracle)


@pytest.mark.parametrize("causal", [False, True])
def test_row_stats_match_full_oracle(causal):
    q, k, v, do = (rand((1, 1, 70, 8), s) for s in (90, 91, 92, 93))
    O, L = attention_forward(q, k, v, causal, 0.3)
    Lr, Dr = attention_row_stats(q[0, 0], k[0, 0], v[0, 0], do[0, 0], causal, 0.3, block=16)
    assert np.allclose(Lr, L[0, 0], atol=1e-13)
    assert np.allclose(Dr, np.sum(do[0, 0] * O[0, 0], axis=1), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_key_rows_match_full_backward_and_autograd(causal):
    """dK, dV of sampled key rows equal those rows of the full analytic backward and of torch
    float64 autograd; with every key selected they are the whole gradient."""
    N, d = 53, 8
    q, k, v, do = (rand((1, 1, N, d), s) for s in (94, 95, 96, 97))
    O, L = attention_forward(q, k, v, causal, 0.45)
    _, dk, dv = attention_backward(q, k, v, O, L, do, causal, 0.45)
    tq, tk, tv = (torch.from_numpy(a).requires_grad_() for a in (q, k, v))
    torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal,
                                                     scale=0.45).backward(torch.from_numpy(do))
    for keys in (np.array([0, 1, 17, 51, 52]), np.arange(N)):
        dk_r, dv_r = attention_dkdv_key_rows(q[0, 0], k[0, 0], v[0, 0], do[0, 0], keys, causal,
                                             0.45)
        assert np.allclose(dk_r, dk[0, 0, keys], atol=1e-12)
        assert np.allclose(dv_r, dv[0, 0, keys], atol=1e-12)
        assert np.allclose(dk_r, tk.grad.numpy()[0, 0, keys], atol=1e-12)
        assert np.allclose(dv_r, tv.grad.numpy()[0, 0, keys], atol=1e-12)


def test_key_rows_invariants_and_closed_forms():
    """Over all keys, sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i; causal: the last key is seen
    only by the last query, so dV_{N-1} = P_{N-1,N-1} dO_{N-1}; with Q = 0 that weight is 1/N."""
    N, d = 40, 4
    q, k, v, do = (rand((N, d), s) for s in (98, 99, 100, 101))
    keys = np.arange(N)
    for causal in (False, True):
        dk, dv = attention_dkdv_key_rows(q, k, v, do, keys, causal, 0.5)
        assert np.allclose(dk.sum(axis=0), 0.0, atol=1e-12)
        assert np.allclose(dv.sum(axis=0), do.sum(axis=0), atol=1e-12)
    _, dv_last = attention_dkdv_key_rows(np.zeros((N, d)), k, v, do, np.array([N - 1]), True, 0.5)
    assert np.allclose(dv_last[0], do[N - 1] / N, atol=1e-15)


@pytest.mark.parametrize("slip", ["no_D", "key_mask_transposed", "unscaled_dk"])
def test_key_rows_planted_mistakes_fail(slip):
    """Broken copies of the key-row function disagree with torch float64 autograd."""
    N, d = 23, 4
    q, k, v, do = (rand((N, d), s) for s in (102, 103, 104, 105))
    keys = np.array([0, 5, 22])
    tq, tk, tv = (torch.from_numpy(a[None, None]).requires_grad_() for a in (q, k, v))
    torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True,
                                                     scale=0.6).backward(
        torch.from_numpy(do[None, None]))
    L, D = attention_row_stats(q, k, v, do, True, 0.6)
    if slip == "no_D":
        dk, dv = attention_dkdv_key_rows(q, k, v, do, keys, True, 0.6, stats=(L, 0 * D))
    elif slip == "key_mask_transposed":
        dk, dv = attention_dkdv_key_rows(q[::-1], k, v, do[::-1], keys, True, 0.6,
                                         stats=(L[::-1], D[::-1]))
    else:
        dk, dv = attention_dkdv_key_rows(q, k, v, do, keys, True, 0.6)
        dk = dk / 0.6
    ok = (np.allclose(dk, tk.grad.numpy()[0, 0, keys], atol=1e-9) and
          np.allclose(dv, tv.grad.numpy()[0, 0, keys], atol=1e-9))
    assert not ok
