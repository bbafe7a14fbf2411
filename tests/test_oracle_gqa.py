"""Pins for the grouped-query (GQA / MQA) oracle functions, against facts that do not come from the
oracle itself: a brute-force loop over single query rows that reads key/value head h // G as the
library header and the oracle define it, and central finite differences of the loss for the
gradients.  Planted mistakes at the end (the head mapping as h % H_kv, a missing or misordered sum
over the group) must each fail a pin.
"""
import math

import numpy as np
import pytest

from oracle import attention_backward_gqa, attention_forward_gqa


def rand(shape, seed, sigma=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * sigma


def _row_brute_force(q, k, v, b, h, i, G, causal, scale):
    """One query row of one head with explicit loops: key/value head h // G."""
    hk = h // G
    N, d = k.shape[2], k.shape[3]
    scores = []
    for j in range(N):
        if causal and j > i:
            continue
        scores.append((j, scale * sum(q[b, h, i, c] * k[b, hk, j, c] for c in range(d))))
    m = max(s for _, s in scores)
    w = [(j, math.exp(s - m)) for j, s in scores]
    z = sum(e for _, e in w)
    o = [sum(e * v[b, hk, j, c] for j, e in w) / z for c in range(v.shape[3])]
    return o, m + math.log(z)


def pin_gqa_forward_brute_force(fwd, bwd):
    for (B, H, Hkv, N, d, seed) in ((1, 4, 2, 5, 3, 1), (2, 6, 3, 4, 2, 2), (1, 3, 1, 6, 3, 3),
                                    (1, 2, 2, 3, 4, 4)):
        q = rand((B, H, N, d), seed)
        k = rand((B, Hkv, N, d), seed + 100)
        v = rand((B, Hkv, N, d), seed + 200)
        for causal in (False, True):
            O, L = fwd(q, k, v, causal, 0.7)
            for b in range(B):
                for h in range(H):
                    for i in range(N):
                        o, l = _row_brute_force(q, k, v, b, h, i, H // Hkv, causal, 0.7)
                        if not (np.allclose(O[b, h, i], o, atol=1e-12) and abs(L[b, h, i] - l) < 1e-12):
                            return f"forward row ({b},{h},{i}) disagrees (H={H}, H_kv={Hkv})"
    return None


def _fd_grads(q, k, v, do, causal, scale, fwd, h=1e-6):
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
            g[idx] = (np.sum(fwd(*plus, causal, scale)[0] * do) -
                      np.sum(fwd(*minus, causal, scale)[0] * do)) / (2 * h)
        grads.append(g)
    return grads


def pin_gqa_backward_finite_differences(fwd, bwd):
    for (H, Hkv, N, d, seed) in ((4, 2, 4, 3, 11), (3, 1, 3, 2, 12), (4, 4, 3, 2, 13)):
        q = rand((1, H, N, d), seed)
        k = rand((1, Hkv, N, d), seed + 1)
        v = rand((1, Hkv, N, d), seed + 2)
        do = rand((1, H, N, d), seed + 3)
        for causal in (False, True):
            O, L = fwd(q, k, v, causal, 0.6)
            got = bwd(q, k, v, O, L, do, causal, 0.6)
            want = _fd_grads(q, k, v, do, causal, 0.6, fwd)
            for name, a, b in zip(("dq", "dk", "dv"), got, want):
                if a.shape != b.shape or not np.allclose(a, b, rtol=1e-6, atol=1e-8):
                    return f"{name} != finite differences (H={H}, H_kv={Hkv}, causal={causal})"
    return None


PINS = [pin_gqa_forward_brute_force, pin_gqa_backward_finite_differences]


def run_pins(fwd, bwd):
    return [m for m in (p(fwd, bwd) for p in PINS) if m]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_gqa_pin(pin):
    assert pin(attention_forward_gqa, attention_backward_gqa) is None


def test_gqa_rejects_non_dividing_heads():
    with pytest.raises(ValueError):
        attention_forward_gqa(rand((1, 3, 2, 2), 0), rand((1, 2, 2, 2), 1), rand((1, 2, 2, 2), 2),
                              False, 1.0)


# --------------------------------------------------------------------------------------------
# planted mistakes (each a plausible slip in the grouped oracle)

def _mut_fwd_tiled(q, k, v, causal, scale):
    """Head mapping h % H_kv (np.tile) instead of h // G."""
    from oracle import attention_forward
    G = q.shape[1] // k.shape[1]
    return attention_forward(q, np.tile(k, (1, G, 1, 1)), np.tile(v, (1, G, 1, 1)), causal, scale)


def _mut_bwd_first_head_only(q, k, v, o, lse, do, causal, scale):
    """dK, dV of the first query head of each group instead of the group's sum."""
    from oracle import attention_backward
    G = q.shape[1] // k.shape[1]
    dq, dk, dv = attention_backward(q, np.repeat(k, G, 1), np.repeat(v, G, 1), o, lse, do, causal,
                                    scale)
    return dq, dk[:, ::G], dv[:, ::G]


def _mut_bwd_sum_misordered(q, k, v, o, lse, do, causal, scale):
    """Group sum over the wrong axis order (heads interleaved as h % H_kv)."""
    from oracle import attention_backward
    B, Hkv, N, d = k.shape
    G = q.shape[1] // Hkv
    dq, dk, dv = attention_backward(q, np.repeat(k, G, 1), np.repeat(v, G, 1), o, lse, do, causal,
                                    scale)
    return (dq, dk.reshape(B, G, Hkv, N, d).sum(axis=1), dv.reshape(B, G, Hkv, N, d).sum(axis=1))


MUTANTS = [
    ("fwd_mapping_tiled", _mut_fwd_tiled, attention_backward_gqa),
    ("bwd_first_head_only", attention_forward_gqa, _mut_bwd_first_head_only),
    ("bwd_sum_misordered", attention_forward_gqa, _mut_bwd_sum_misordered),
]


@pytest.mark.parametrize("name,fwd,bwd", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_gqa_planted_mistake_is_caught(name, fwd, bwd):
    assert run_pins(fwd, bwd), f"planted mistake {name} passed every pin"
